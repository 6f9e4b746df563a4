"""C-ABI library checks that need no GPU: it loads, exports every symbol that
include/gmla.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "gmla.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"GMLA_API\s+[\w\s\*]+?\b(gmla_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def gmla():
    from causal_head_latent_b200 import build
    build.build()
    import causal_head_latent_b200 as g
    return g


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for name in ("gmla_latent_project", "gmla_attend_prefill", "gmla_attend_decode", "gmla_gate_out"):
        assert name in syms
    assert len(syms) >= 10


def test_library_exports_every_declared_symbol(gmla):
    out = subprocess.run(["nm", "-D", "--defined-only", gmla.library_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gmla_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(gmla.lib, name)
    # nothing else leaks from the library's C++ internals
    assert not [s for s in re.findall(r"\bT (\S+)", out) if "gmla" in s and not s.startswith("gmla_")]


def test_status_strings_and_version(gmla):
    for code in range(6):
        assert gmla.gmla_status_string(code)
    assert gmla.gmla_version() >= 100


def _i3(*v):
    return (ctypes.c_int64 * 3)(*v)


def test_host_validation_without_gpu(gmla):
    L = gmla.lib
    fake = 0x10000  # never dereferenced: every call below fails validation first
    s = _i3(128 * 2 * 300, 128 * 2, 128)
    # null Q
    assert L.gmla_attend_prefill(None, s, fake, s, fake, s, 1, 2, 300, 300, 128, 1, 0.0, None, fake, s, None, None,
                                 None) == 1
    # Tq > Tk
    assert L.gmla_attend_prefill(fake, s, fake, s, fake, s, 1, 2, 301, 300, 128, 1, 0.0, None, fake, s, None, None,
                                 None) == 1
    # causal flag not boolean
    assert L.gmla_attend_prefill(fake, s, fake, s, fake, s, 1, 2, 300, 300, 128, 2, 0.0, None, fake, s, None, None,
                                 None) == 1
    # misaligned pointer
    assert L.gmla_attend_prefill(fake + 2, s, fake, s, fake, s, 1, 2, 300, 300, 128, 1, 0.0, None, fake, s, None,
                                 None, None) == 1
    # stride not a multiple of 8 elements
    assert L.gmla_attend_prefill(fake, _i3(100, 12, 4), fake, s, fake, s, 1, 2, 300, 300, 128, 1, 0.0, None, fake, s,
                                 None, None, None) == 1
    # head width other than 128
    assert L.gmla_attend_prefill(fake, s, fake, s, fake, s, 1, 2, 300, 300, 64, 1, 0.0, None, fake, s, None, None,
                                 None) == 2
    # latent project: cache too short, K requested without C, d_model not a multiple of 128
    assert L.gmla_latent_project(fake, 2, 10, 256, fake, fake, fake, 64, fake, fake, fake, fake, fake, 15, 6, None,
                                 None, None) == 1
    assert L.gmla_latent_project(fake, 2, 10, 256, fake, fake, fake, 64, fake, fake, fake, fake, None, 16, 0, fake,
                                 None, None) == 1
    assert L.gmla_latent_project(fake, 2, 10, 200, fake, fake, fake, 64, fake, fake, fake, fake, fake, 16, 0, None,
                                 None, None) == 2
    # head-range projections: empty range, range past the heads
    LPH = L.gmla_latent_project_heads
    assert LPH(fake, 2, 10, 256, 1, 1, fake, fake, fake, 64, fake, fake, fake, fake, fake, 16, 0, None, None,
               None) == 1
    assert LPH(fake, 2, 10, 256, 1, 3, fake, fake, fake, 64, fake, fake, fake, fake, fake, 16, 0, None, None,
               None) == 1
    # decode: L beyond the cache, and a short workspace
    assert L.gmla_attend_decode(fake, fake, 2, 100, 101, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 1 << 30,
                                None) == 1
    assert L.gmla_attend_decode(fake, fake, 2, 100, 100, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 16,
                                None) == 5
    assert L.gmla_attend_decode_workspace_size(2, 100, 2, 64) > 16
    # varlen decode: null lens, a zero length, a length past the cache, a short workspace
    lens = (ctypes.c_int64 * 2)(5, 7)
    bad0 = (ctypes.c_int64 * 2)(5, 0)
    bad1 = (ctypes.c_int64 * 2)(5, 101)
    LV = L.gmla_attend_decode_varlen
    assert LV(fake, fake, 2, 100, None, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 1 << 30, None) == 1
    assert LV(fake, fake, 2, 100, bad0, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 1 << 30, None) == 1
    assert LV(fake, fake, 2, 100, bad1, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 1 << 30, None) == 1
    assert LV(fake, fake, 2, 100, lens, 2, 128, 64, fake, fake, 0.0, None, fake, None, fake, 16, None) == 5
    assert L.gmla_attend_decode_varlen_workspace_size(2, 100, 2, 64) > L.gmla_attend_decode_workspace_size(2, 100, 2,
                                                                                                          64)
    # varlen prefill: q_len > kv_len, kv_len 0, a short workspace
    PV = L.gmla_attend_prefill_varlen
    ql, kl = (ctypes.c_int64 * 2)(10, 20), (ctypes.c_int64 * 2)(20, 20)
    qbad, kbad = (ctypes.c_int64 * 2)(21, 20), (ctypes.c_int64 * 2)(20, 0)
    for qq, kk, ws, code in ((qbad, kl, 1 << 20, 1), (ql, kbad, 1 << 20, 1), (ql, kl, 8, 5)):
        assert PV(fake, s, fake, s, fake, s, 2, 2, 300, 300, 128, qq, kk, 1, 0.0, None, fake, s, None, fake, ws,
                  None) == code
    # varlen prefill: misaligned workspace; head width other than 128
    assert PV(fake, s, fake, s, fake, s, 2, 2, 300, 300, 128, ql, kl, 1, 0.0, None, fake, s, None, fake + 8, 1 << 20,
              None) == 1
    assert PV(fake, s, fake, s, fake, s, 2, 2, 300, 300, 64, ql, kl, 1, 0.0, None, fake, s, None, fake, 1 << 20,
              None) == 2
    # varlen decode: more than 96 heads, d_c not a multiple of 64
    assert LV(fake, fake, 2, 100, lens, 97, 128, 64, fake, fake, 0.0, None, fake, None, fake, 1 << 30, None) == 2
    assert LV(fake, fake, 2, 100, lens, 2, 128, 96, fake, fake, 0.0, None, fake, None, fake, 1 << 30, None) == 2
    # expand_kv: range past the cache, no output, d_model not a multiple of 128
    assert L.gmla_expand_kv(fake, 2, 100, 50, 51, 64, fake, fake, 256, fake, fake, None) == 1
    assert L.gmla_expand_kv(fake, 2, 100, 0, 10, 64, fake, fake, 256, None, None, None) == 1
    assert L.gmla_expand_kv(fake, 2, 100, 0, 10, 64, fake, fake, 200, fake, fake, None) == 2
    # an empty query set is a no-op that launches nothing
    assert L.gmla_attend_prefill(fake, s, fake, s, fake, s, 1, 2, 0, 300, 128, 1, 0.0, None, fake, s, None, None,
                                 None) == 0
    # the timeout self-test refuses limits outside 1..1000 ms
    assert L.gmla_selftest_wait_timeout(0, None) == 1
    assert L.gmla_selftest_wait_timeout(5000, None) == 1
    # gate_out: a gate needs a workspace for the gated context; bad pointers and head ranges
    assert L.gmla_gate_out(fake, fake, fake, 4, 256, fake, None, 0, None) == 5
    need = L.gmla_gate_out_workspace_size(4, 256)
    assert need >= 4 * 256 * 2
    assert L.gmla_gate_out(fake, fake, fake, 4, 256, fake, fake, need - 1, None) == 5
    assert L.gmla_gate_out(None, None, fake, 4, 256, fake, None, 0, None) == 1
    assert L.gmla_gate_out(fake, None, fake, 4, 200, fake, None, 0, None) == 2
    assert L.gmla_gate_out_heads(fake, None, fake, 4, 256, 0, 3, fake, None, 0, None) == 1
    assert L.gmla_gate_out_heads(fake, None, fake, 4, 256, 2, 1, fake, None, 0, None) == 1
    # partial decode: bad key ranges, a short workspace; combine: no parts, too many parts
    PD = L.gmla_attend_decode_partial
    assert PD(fake, fake, 2, 100, 50, 40, 2, 128, 64, fake, 0.0, fake, fake, fake, 1 << 30, None) == 1
    assert PD(fake, fake, 2, 100, 0, 101, 2, 128, 64, fake, 0.0, fake, fake, fake, 1 << 30, None) == 1
    assert PD(fake, fake, 2, 100, 10, 60, 2, 128, 64, fake, 0.0, fake, fake, fake, 16, None) == 5
    assert PD(fake, fake, 2, 100, 10, 60, 2, 128, 64, fake, 0.0, None, fake, fake, 1 << 30, None) == 1
    assert L.gmla_attend_decode_partial_workspace_size(2, 10, 60, 2, 64) > 16
    assert L.gmla_attend_decode_partial_workspace_size(2, 10, 10, 2, 64) == 0
    assert L.gmla_decode_combine(fake, fake, 0, 2, 2, 128, 64, fake, None, fake, None) == 1
    assert L.gmla_decode_combine(fake, fake, 1025, 2, 2, 128, 64, fake, None, fake, None) == 2
    assert L.gmla_decode_combine(fake, fake, 2, 2, 2, 128, 96, fake, None, fake, None) == 2


def test_binding_has_no_cpu_path():
    import causal_head_latent_b200 as g
    src = open(os.path.join(ROOT, "causal_head_latent_b200", "__init__.py")).read()
    assert "oracle" not in src and "numpy" not in src
    assert callable(g.gmla_attend_prefill)
