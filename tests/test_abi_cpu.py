"""The C-ABI library loads on a CPU-only host, exports every symbol the header
declares, and rejects invalid arguments with a status before any launch."""
import ctypes as C
import re
from pathlib import Path

import pytest
import torch

import kernelized_linear_attention_chunked_b200 as kata
from kernelized_linear_attention_chunked_b200 import _binding

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "kata.h"


def header_functions():
    text = HEADER.read_text()
    return re.findall(r"KATA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_symbols_exported_and_bound():
    names = header_functions()
    assert len(names) == 32
    L = kata.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_binding.SIGNATURES)


def test_header_argument_counts_match_binding():
    text = HEADER.read_text()
    for name, (_, args) in _binding.SIGNATURES.items():
        m = re.search(r"KATA_API[^;(]*\b" + name + r"\(([^)]*)\)", text)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), name


def test_status_strings_and_helpers():
    L = kata.lib()
    assert L.kata_version() >= 100
    assert L.kata_status_string(0) == b"KATA_OK"
    assert L.kata_status_string(4) == b"KATA_ERR_TIMEOUT"
    assert L.kata_status_string(6) == b"KATA_ERR_BOUNDS"
    assert L.kata_status_string(99) == b"KATA_ERR_UNKNOWN"
    assert kata.launch_count() == 0  # validation failures launch nothing
    for d in (16, 32, 64):
        assert kata.packed_dim(d) == d * (d + 1) // 2


def test_workspace_holds_segment_partial_states():
    # a final-state-only bf16 call of one head over two 128-token chunks splits
    # the sequence in two segments: their partial states must fit
    L = kata.lib()
    d, D = 32, 32 * 33 // 2
    align = lambda x: (x + 255) // 256 * 256
    parts = align(2 * D * d * 4) + align(2 * D * 4)
    s_copy = align(D * 4)
    assert L.kata_prefill_workspace_bytes(1, 1, 256, d, 64, 1) >= s_copy + parts


def test_workspace_queries():
    L = kata.lib()
    assert L.kata_prefill_workspace_bytes(1, 1, 256, 16, 64, 0) > 0
    assert L.kata_prefill_workspace_bytes(1, 1, 250, 16, 64, 0) == 0  # T not a multiple
    assert L.kata_prefill_workspace_bytes(1, 1, 256, 24, 64, 0) == 0  # d not built
    assert L.lola_sre_workspace_bytes(2, 8, 64, 192) > 0
    assert L.lola_sre_workspace_bytes(2, 8, 64, 2000) == 0
    assert L.lola_prefill_workspace_bytes(2, 8, 8192, 64, 64, 128) > 0
    assert L.kata_prefill_path(1, 1, 256, 16, 64, 0) == 0  # fp32: CUDA cores
    assert L.kata_prefill_path(1, 1, 250, 16, 64, 0) == -1
    big = L.kata_prefill_host_workspace_bytes(1, 1, 256, 16, 64, 0)
    assert big >= 4 * 256 * 16 * 4


FAKE = C.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
MISALIGNED = C.c_void_p((1 << 20) + 4)


def _prefill(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=0, B=1, H=1, T=256, d=16, chunk=64, eps=1e-6,
             H_in=None, s_in=None, o=FAKE, H_out=None, s_out=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return kata.lib().kata_prefill(*a.values(), None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1),
    (dict(k=MISALIGNED), 1),
    (dict(d=24), 2),
    (dict(chunk=48), 2),
    (dict(T=250), 1),
    (dict(B=0), 1),
    (dict(dtype=7), 2),
    (dict(eps=-1.0), 1),
    (dict(H_in=FAKE), 1),  # s_in missing
    (dict(ws=None, ws_bytes=0), 5),
])
def test_prefill_validation(kw, status):
    assert _prefill(**kw) == status
    assert kata.lib().kata_last_error()


def _prefill_ex(form, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, B=1, H=1, T=256, d=32, chunk=64, eps=1e-6,
             H_in=None, s_in=None, o=FAKE, H_out=None, s_out=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return kata.lib().kata_prefill_ex(*a.values(), None, form)


def test_prefill_form_selection():
    L = kata.lib()
    assert L.kata_quadratic_max_tokens(32) >= 2048
    assert L.kata_quadratic_max_tokens(16) == 0
    for d in (32, 64):
        tmax = L.kata_quadratic_max_tokens(d)
        assert tmax % 128 == 0
        # output-only bf16 calls up to the crossover take the quadratic form
        assert L.kata_prefill_auto_form(4, 8, tmax, d, 64, 1, 0) == 2
        assert L.kata_prefill_auto_form(4, 8, tmax + 128, d, 64, 1, 0) == 1
        # with an initial or final state, fp32 inputs, or T % 128 != 0: chunked
        assert L.kata_prefill_auto_form(4, 8, 1024, d, 64, 1, 1) == 1
        assert L.kata_prefill_auto_form(4, 8, 1024, d, 64, 0, 0) == 1
        assert L.kata_prefill_auto_form(4, 8, 192, d, 64, 1, 0) == 1
    assert L.kata_prefill_auto_form(1, 1, 256, 16, 64, 1, 0) == 1
    assert L.kata_prefill_auto_form(1, 1, 250, 32, 64, 1, 0) == -1
    assert kata.prefill_auto_form(4, 8, 2048, 32, 64, torch.bfloat16) == "quadratic"
    assert kata.prefill_auto_form(4, 8, 2048, 32, 64, torch.bfloat16, True) == "chunked"
    assert kata.prefill_auto_form(2, 16, 16384, 64, 128, torch.bfloat16) == "chunked"


@pytest.mark.parametrize("form,kw,status", [
    (7, {}, 1),                                    # no such form
    (-1, {}, 1),
    (2, dict(dtype=0), 2),                         # quadratic: bf16 only
    (2, dict(d=16), 2),                            # quadratic: d = 32 or 64
    (2, dict(T=192), 2),                           # quadratic: T a multiple of 128
    (2, dict(o=None, H_out=FAKE, s_out=FAKE), 2),  # quadratic: o is required
    (2, dict(H_in=FAKE, s_in=FAKE), 2),             # quadratic: zero initial state only
    (2, dict(q=MISALIGNED), 1),
    (1, dict(ws=None, ws_bytes=0), 5),             # the chunked form needs its workspace
])
def test_prefill_ex_validation(form, kw, status):
    assert _prefill_ex(form, **kw) == status
    assert kata.lib().kata_last_error()


def test_decode_and_lola_validation():
    L = kata.lib()
    assert L.kata_decode_step(FAKE, FAKE, FAKE, 1, 2, 2, 48, 1e-6, FAKE, FAKE, FAKE, None) == 2
    assert L.kata_decode_step(FAKE, None, FAKE, 1, 2, 2, 64, 1e-6, FAKE, FAKE, FAKE, None) == 1
    assert L.lola_sre_score_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 64, 0, 4, 1e-6, 0,
                                 None, FAKE, None, None, FAKE, 1 << 30, None) == 1
    assert L.lola_sre_score_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 64, 8, 4, 1e-6, 1,
                                 None, FAKE, None, None, FAKE, 1 << 30, None) == 1
    assert L.lola_hybrid_readout(FAKE, FAKE, FAKE, 1, 1, 1, 128, 64, 64, 64, 80, FAKE, FAKE, 0,
                                 8, FAKE, FAKE, 1e-6, 0.125, FAKE, FAKE, 1 << 30, None) == 1
    assert L.lola_prefill(FAKE, FAKE, FAKE, 1, 1, 1, 100, 64, 64, 8, 1e-6, 0.125, FAKE, FAKE,
                          FAKE, None, FAKE, 1 << 30, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "LIB_PATH", tmp_path / "missing.so")
    with pytest.raises(kata.KataError):
        _binding.lib()


def test_forced_timeout_hook_validation():
    L = kata.lib()
    # quadratic form only (d = 32 or 64, T a multiple of 128); polls in [1, 2^20]
    assert L.kata_test_forced_timeout(FAKE, FAKE, FAKE, 1, 1, 256, 16, 1e-6, FAKE, 64, None) == 2
    assert L.kata_test_forced_timeout(FAKE, FAKE, FAKE, 1, 1, 192, 32, 1e-6, FAKE, 64, None) == 1
    assert L.kata_test_forced_timeout(FAKE, FAKE, FAKE, 1, 1, 256, 32, 1e-6, FAKE, 0, None) == 1
    assert L.kata_test_forced_timeout(FAKE, FAKE, FAKE, 1, 1, 256, 32, 1e-6, FAKE, 1 << 21,
                                      None) == 1
    assert L.kata_test_forced_timeout(FAKE, None, FAKE, 1, 1, 256, 32, 1e-6, FAKE, 64, None) == 1
    assert kata.launch_count() == 0


def test_feature_dims_and_validation():
    L = kata.lib()
    assert L.kata_feature_dim(64, 0, 1) == 2080
    assert L.kata_feature_dim(64, 1, 2) == 2 * 528
    assert L.kata_feature_dim(64, 2, 2) == 528
    assert L.kata_feature_dim(64, 1, 8) == 8 * 36
    assert L.kata_feature_dim(32, 2, 4) == 36
    assert L.kata_feature_dim(64, 0, 2) == 0   # the rank-one feature has g = 1
    assert L.kata_feature_dim(64, 1, 16) == 0  # factors of 4 values: too small
    assert L.kata_feature_dim(48, 1, 2) == 0   # d not built
    assert L.kata_feature_dim(64, 3, 2) == 0
    # bad feature / g are refused before any launch
    args = (FAKE, FAKE, FAKE, 1, 1, 2, 128, 32, 64, 1e-6)
    assert L.kata_prefill_feature(*args, 3, 2, None, None, FAKE, None, None, None, 0, None) == 2
    assert L.kata_prefill_feature(*args, 1, 8, None, None, FAKE, None, None, None, 0, None) == 2
    assert L.kata_prefill_feature(*args, 1, 2, FAKE, None, FAKE, None, None, None, 0, None) == 1
    assert L.kata_decode_step_feature(FAKE, FAKE, FAKE, 1, 1, 1, 32, 1e-6, 2, 3, FAKE, FAKE,
                                      FAKE, None) == 2
    assert kata.launch_count() == 0


def test_bounds_hook_compiled_out_of_the_normal_library():
    L = kata.lib()
    if kata.debug_build():
        pytest.skip("this process loaded the debug library")
    assert L.kata_debug_build() == 0
    assert L.kata_test_bounds_check(None) == 2  # KATA_ERR_UNSUPPORTED, nothing launched
    assert kata.launch_count() == 0


def test_debug_library_loads_and_exports_every_symbol():
    # a separate process: each library carries its own static CUDA runtime
    import os
    import subprocess
    import sys
    lib_debug = ROOT / "kernelized_linear_attention_chunked_b200" / "libkata_debug.so"
    if not lib_debug.exists():
        pytest.skip("libkata_debug.so not built")
    code = (
        "import re, sys; sys.path.insert(0, %r)\n"
        "import kernelized_linear_attention_chunked_b200 as kata\n"
        "from kernelized_linear_attention_chunked_b200 import _binding\n"
        "assert _binding.LIB_PATH.name == 'libkata_debug.so'\n"
        "assert kata.debug_build()\n"
        "names = re.findall(r'KATA_API\\s+[\\w\\s\\*]+?\\b(\\w+)\\s*\\(', open(%r).read())\n"
        "L = kata.lib()\n"
        "assert all(hasattr(L, n) for n in names)\n"
        "print('ok', len(names))\n" % (str(ROOT), str(HEADER)))
    env = dict(os.environ, KATA_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "ok 32"
