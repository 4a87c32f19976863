"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
function include/qmoe.h declares (no compute call is made here)."""
import ctypes
import os
import re

from moe_expert_gemv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "qmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("qgemv_affine", "moe_router_topk", "moe_expert_qmlp", "moe_prefill_qgemm"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(build.build())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, "not exported: %s" % missing


def test_status_strings_without_gpu():
    lib = ctypes.CDLL(build.build())
    lib.qmoe_status_string.restype = ctypes.c_char_p
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert lib.qmoe_status_string(code).startswith(b"QMOE_")
