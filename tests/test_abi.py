"""The C-ABI library loads and exports every function include/thdcp.h declares, and
the Python binding declares exactly those.  No compute calls: CPU only."""
import ctypes
import os
import re
import subprocess

from context_packed_sequence_cp_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "thdcp.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[\w\s\*]*?\b(thd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("thd_cp_plan", "thd_kv_gather", "thd_cp_attn_fwd", "thd_cp_attn_bwd"):
        assert want in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(_lib.LIB_PATH)
    for name in _declared():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (thd_\w+)", out))
    assert set(_declared()) <= exported


def test_binding_covers_the_header():
    assert sorted(_lib.SIGNATURES) == _declared()


def test_strerror_texts():
    L = _lib.lib()
    for code in list(_lib.ERRORS) + [0]:
        assert L.thd_cp_strerror(code)
