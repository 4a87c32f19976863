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


def test_binding_status_codes_match_the_header():
    """The binding's ERR_* constants carry the values of the header's enum."""
    from moe_expert_gemv_b200 import qmoe
    src = open(os.path.join(ROOT, "include", "qmoe.h")).read()
    codes = dict(re.findall(r"QMOE_(ERR_[A-Z_]+)\s*=\s*(-?\d+)", src))
    assert len(codes) == 7
    for name, value in codes.items():
        assert getattr(qmoe, name) == int(value), name


def test_one_pass_workspace_sizes_without_gpu():
    """qgemv_affine_workspace_bytes is host arithmetic: the one-pass plan for
    batch 9..32 (K slices whose x fits 64 KB of shared memory, ~32 KB weight
    tiles) and its workspace (64 KB of tile counters + fp32 partial tiles)."""
    lib = ctypes.CDLL(build.build())
    f = lib.qgemv_affine_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int32] * 4
    # batch <= 8, an unsupported width (rows of 96 bytes) or bad arguments: none
    assert f(14336, 4096, 4, 8) == 0
    assert f(136, 192, 4, 32) == 0
    assert f(14336, 4096, 3, 32) == 0 and f(14336, 4096, 4, 33) == 0 and f(0, 4096, 4, 16) == 0
    # x of 32 x 1024 fp16 = 64 KB: one slice, no workspace
    assert f(512, 1024, 4, 32) == 0
    # K=4096, batch 32: 4 slices of 1024, 64-row tiles, 4 n-tiles of 8 columns
    tiles = 14336 // 64
    assert f(14336, 4096, 4, 32) == 65536 + tiles * 4 * (4 * 4 * 32) * 16
    # batch 16: 2 slices of 2048 (64 KB of x), 32-row tiles (1 KB of codes a row), 2 n-tiles
    tiles = 14336 // 32
    assert f(14336, 4096, 4, 16) == 65536 + tiles * 2 * (2 * 2 * 32) * 16
    # batch 9 rounds up to 2 n-tiles; 8-bit rows of 2048 codes: 16-row tiles
    tiles = (1000 + 15) // 16
    assert f(1000, 4096, 8, 9) == 65536 + tiles * 2 * (1 * 2 * 32) * 16
    # K=8192 at batch 32: 8 slices of 1024
    assert f(256, 8192, 4, 32) == 65536 + (256 // 64) * 8 * (4 * 4 * 32) * 16


def test_decode_pack_holds_exactly_the_row_major_bytes_without_gpu():
    """moe_decode_pack_bytes is host arithmetic: the streaming layout is a
    permutation of the row-major layer (8-bit router + E routed experts + the
    shared expert, codes and fp16 scale + bias per 64 inputs), nothing added."""
    from moe_expert_gemv_b200 import qmoe
    lib = ctypes.CDLL(build.build())
    f = lib.moe_decode_pack_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_void_p]

    def mat_bytes(rows, cols, bits):
        return rows * cols * bits // 8 + 2 * rows * (cols // 64) * 2

    for E, H, I in ((128, 2816, 704), (16, 256, 64), (64, 1024, 192)):
        L = qmoe.CMoeLayer()
        L.num_experts, L.hidden, L.inter = E, H, I
        want = mat_bytes(E, H, 8) + (E + 1) * (2 * mat_bytes(I, H, 4) + mat_bytes(H, I, 4))
        assert f(ctypes.addressof(L)) == want
    # the numbers the benchmark quotes: 30 layers of the 128-expert layer
    L = qmoe.CMoeLayer()
    L.num_experts, L.hidden, L.inter = 128, 2816, 704
    assert f(ctypes.addressof(L)) == 382976 + 129 * 3345408
    assert 30 * f(ctypes.addressof(L)) == 12958218240   # "12.96 GB of weights"


def test_header_is_plain_c_and_links_from_c(tmp_path):
    """include/qmoe.h is a C header (strict C11, no C++ constructs), and a C
    program links against the library and calls it (no GPU call)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        import pytest
        pytest.skip("no C compiler")
    lib = build.build()
    src = tmp_path / "use.c"
    src.write_text('#include "qmoe.h"\n#include <string.h>\n'
                   'int main(void) {\n'
                   '  if (qmoe_version() <= 0) return 1;\n'
                   '  if (strncmp(qmoe_status_string(QMOE_OK), "QMOE_", 5)) return 2;\n'
                   '  if (qgemv_affine_workspace_bytes(14336, 4096, 4, 8) != 0) return 3;\n'
                   '  return 0;\n}\n')
    exe = tmp_path / "use"
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", os.path.dirname(lib), "-lqmoe",
                    "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0
