"""The C-ABI library loads without a GPU and exports exactly the entry points that
include/qevict.h declares (no compute calls: nothing here needs a device)."""
from __future__ import annotations

import ctypes
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qevict.h")


def declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    return sorted(set(re.findall(r"QE_API\s+[\w\s\*]*?\b(qe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def libpath():
    from kv_cache_eviction_gqa_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = declared()
    for must in ("qe_create", "qe_kv_append", "qe_decode_attend_and_score", "qe_route_windows",
                 "qe_quantize_once", "qe_promote", "qe_vwo_l1norm", "qe_criticalkv_select",
                 "qe_trim_global_topm", "qe_decode_attend_and_score_noalloc", "qe_diag_tiers",
                 "qe_diag_fmm"):
        assert must in names


def test_every_declared_symbol_is_exported(libpath):
    L = ctypes.CDLL(libpath)
    missing = [n for n in declared() if not hasattr(L, n)]
    assert not missing, f"declared but not exported: {missing}"


@pytest.mark.skipif(shutil.which("nm") is None, reason="nm not available")
def test_no_undeclared_exports(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted({l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("qe_")})
    extra = sorted(set(exported) - set(declared()))
    assert not extra, f"exported but not declared: {extra}"


def test_host_side_argument_errors_need_no_device(libpath):
    from kv_cache_eviction_gqa_b200 import binding as B
    L = B.lib()
    assert L.qe_trim_scratch_bytes(0, 10) == 0
    assert L.qe_trim_scratch_bytes(256, 1536) > 256 * 1536 * 16 * 8
    # null pointers are rejected before anything touches the device
    rc = L.qe_trim_global_topm(None, None, None, None, 1, 1, 1, 128, B.QE_BF16, 10, 1, None, None,
                               None, None, None, None, 0, None)
    assert rc == B.QE_ERR_INVALID_ARG
    assert L.qe_strerror(B.QE_ERR_WORKSPACE).decode() == "workspace too small"
    # diagnostics: sizes and argument checks on the host
    assert L.qe_diag_fmm_scratch_bytes(64, 4) >= 64 * 64 * 4 * 16
    assert L.qe_diag_fmm_scratch_bytes(0, 4) == 0 and L.qe_diag_fmm_scratch_bytes(1, 9) == 0
    assert L.qe_diag_tiers(None, None, None, 1, 1, 0, None, None) == B.QE_ERR_INVALID_ARG
    assert L.qe_diag_fmm(None, None, 1, 0, None, 1, 1, 1, 1, 1, 128, B.QE_BF16, None, None, 0,
                         None) == B.QE_ERR_INVALID_ARG
    # global routing: sizes and argument checks on the host
    assert L.qe_route_global_scratch_bytes(32, 8, 8, 1025) >= 32 * 8 * 8 * 1025 * 10
    assert L.qe_route_global_scratch_bytes(0, 8, 8, 1025) == 0
    assert L.qe_route_windows_global(None, 1, 1, 1, 0.5, None, 0, None) == B.QE_ERR_INVALID_ARG


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_is_plain_c(tmp_path):
    """include/qevict.h is a C header: it compiles as strict C99 (no torch or C++ types)."""
    src = tmp_path / "use.c"
    src.write_text('#include "qevict.h"\n'
                   "int main(void) {\n"
                   "  qe_config c; qe_layout l; (void)c; (void)l;\n"
                   "  return (int)qe_diag_fmm_scratch_bytes(1, 4) + (int)qe_route_global_scratch_bytes(1, 1, 1, 1)\n"
                   "         + (int)qe_trim_scratch_bytes(1, 1);\n"
                   "}\n")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o", str(tmp_path / "use.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_sekv_host_side_sizes_and_errors(libpath):
    from kv_cache_eviction_gqa_b200 import binding as B
    L = B.lib()
    # the state holds summaries for up to (n + 1) / 2 spans per (sequence, kv head) in float32
    n, D = 32768, 128
    assert L.qe_sekv_state_bytes(8, 32, 8, n, D) >= 8 * 8 * ((n + 1) // 2) * D * 4 * 2
    assert L.qe_sekv_state_bytes(1, 4, 1, n, 96) == 0          # D = 96 unsupported
    assert L.qe_sekv_state_bytes(1, 6, 4, n, 128) == 0         # Hq not a multiple of Hkv
    assert L.qe_sekv_state_bytes(1, 4, 1, 0, 128) == 0         # no token
    import ctypes as C
    off = (C.c_size_t * 8)()
    assert L.qe_sekv_state_offsets(2, 8, 2, 1001, 64, off) == B.QE_OK and off[7] == 501
    assert list(off[:7]) == sorted(off[:7])
    assert L.qe_sekv_build(None, None, None, 1, 4, 1, 16, 128, B.QE_BF16, 1.0, None, 0, None) == B.QE_ERR_INVALID_ARG
    assert L.qe_sekv_attend(None, None, None, 1, 4, 1, 16, 128, B.QE_BF16, 1.0, None, 0, None,
                            None) == B.QE_ERR_INVALID_ARG


def test_state_checkpoint_host_checks():
    """qe_state_bytes is the header plus the whole workspace; export before a prefill is out of
    order and touches nothing (stand-in device addresses)."""
    import ctypes as C
    from kv_cache_eviction_gqa_b200 import binding as Bd
    assert Bd.lib().qe_state_bytes(None) == 0
    cfg = Bd.QeConfig(2, 8, 2, 64, Bd.QE_FP16, 16, 16, 8, 8, 0.5, 4, 512, 2048, 2048 // 16 + 4, 16, 16)
    lay = Bd.QeLayout()
    assert Bd.lib().qe_plan(C.byref(cfg), C.byref(lay)) == 0
    h = C.c_void_p()
    fake = C.c_void_p(1 << 40)
    assert Bd.lib().qe_create(C.byref(cfg), fake, C.c_size_t(lay.total), fake, C.byref(h)) == 0
    try:
        n = Bd.lib().qe_state_bytes(h)
        assert n == 256 + lay.total
        assert Bd.lib().qe_state_export(h, fake, C.c_size_t(n), None) == Bd.QE_ERR_STATE
    finally:
        Bd.lib().qe_destroy(h)
