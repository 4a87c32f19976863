"""Host-side validation of the C ABI: every bad argument returns a status and
enqueues nothing.  Calls go through ctypes with raw pointers."""
import ctypes

import pytest
import torch

from moe_expert_gemv_b200 import qmoe

pytestmark = pytest.mark.gpu

INVALID, ALIGN, UNSUP, WS = -1, -2, -3, -7


def mat(rows, cols, bits=4, group=64, off=0):
    P = torch.zeros(rows * cols * bits // 32 + 16, dtype=torch.int32, device="cuda")
    S = torch.zeros(rows * cols // 64 + 16, dtype=torch.float16, device="cuda")
    B = torch.zeros_like(S)
    keep = (P, S, B)
    c = qmoe.CQMatrix(P.data_ptr() + off, S.data_ptr(), B.data_ptr(), rows, cols, bits, group)
    return c, keep


def call_qgemv(c, x, batch, y):
    return qmoe.lib().qgemv_affine(ctypes.byref(c), ctypes.c_void_p(x), batch, ctypes.c_void_p(y),
                                   None, None)


def call_qgemv_ws(c, x, batch, y, ws, nbytes):
    return qmoe.lib().qgemv_affine_ws(ctypes.byref(c), ctypes.c_void_p(x), batch, ctypes.c_void_p(y),
                                      ctypes.c_void_p(ws), nbytes, None, None)


def test_qgemv_ws_argument_errors(cuda_dev):
    rows, cols = 64, 4096
    x = torch.zeros(32 * cols, dtype=torch.float16, device="cuda")
    y = torch.zeros(32 * rows, dtype=torch.float16, device="cuda")
    good, k1 = mat(rows, cols)
    need = qmoe.lib().qgemv_affine_workspace_bytes(rows, cols, 4, 32)
    assert need > 0
    ws = torch.zeros(need + 64, dtype=torch.uint8, device="cuda")
    assert call_qgemv_ws(good, x.data_ptr(), 32, y.data_ptr(), ws.data_ptr(), need) == 0
    assert call_qgemv_ws(good, x.data_ptr(), 32, y.data_ptr(), None, 0) == INVALID
    assert call_qgemv_ws(good, x.data_ptr(), 32, y.data_ptr(), ws.data_ptr(), need - 16) == INVALID
    assert call_qgemv_ws(good, x.data_ptr(), 32, y.data_ptr(), ws.data_ptr() + 8, need) == ALIGN
    assert call_qgemv_ws(good, x.data_ptr(), 33, y.data_ptr(), ws.data_ptr(), need) == INVALID
    # batch <= 8 needs no workspace
    assert call_qgemv_ws(good, x.data_ptr(), 8, y.data_ptr(), None, 0) == 0
    assert qmoe.lib().qgemv_affine_workspace_bytes(rows, cols, 3, 32) == 0
    assert qmoe.lib().qgemv_affine_workspace_bytes(rows, cols, 4, 0) == 0
    torch.cuda.synchronize()


def test_qgemv_argument_errors(cuda_dev):
    x = torch.zeros(8 * 256, dtype=torch.float16, device="cuda")
    y = torch.zeros(8 * 64, dtype=torch.float16, device="cuda")
    good, k1 = mat(64, 256)
    assert call_qgemv(good, x.data_ptr(), 1, y.data_ptr()) == 0
    assert call_qgemv(good, None, 1, y.data_ptr()) == INVALID
    assert call_qgemv(good, x.data_ptr(), 0, y.data_ptr()) == INVALID
    assert call_qgemv(good, x.data_ptr(), 33, y.data_ptr()) == INVALID
    assert call_qgemv(good, x.data_ptr() + 1, 1, y.data_ptr()) == ALIGN
    bad, k2 = mat(64, 256, off=4)
    assert call_qgemv(bad, x.data_ptr(), 1, y.data_ptr()) == ALIGN
    g32, k3 = mat(64, 256, group=32)
    assert call_qgemv(g32, x.data_ptr(), 1, y.data_ptr()) == UNSUP
    b3, k4 = mat(64, 256, bits=3)
    assert call_qgemv(b3, x.data_ptr(), 1, y.data_ptr()) == INVALID
    r12, k5 = mat(12, 256)
    assert call_qgemv(r12, x.data_ptr(), 1, y.data_ptr()) == UNSUP
    torch.cuda.synchronize()


def test_router_and_expert_argument_errors(cuda_dev):
    L = qmoe.lib()
    r, k1 = mat(128, 256, bits=8)
    x = torch.zeros(256, dtype=torch.float16, device="cuda")
    idx = torch.zeros(16, dtype=torch.int32, device="cuda")
    wt = torch.zeros(16, dtype=torch.float32, device="cuda")
    v = ctypes.c_void_p
    assert L.moe_router_topk(ctypes.byref(r), v(x.data_ptr()), 1, 0, v(idx.data_ptr()),
                             v(wt.data_ptr()), None, None, None) == INVALID
    assert L.moe_router_topk(ctypes.byref(r), v(x.data_ptr()), 1, 17, v(idx.data_ptr()),
                             v(wt.data_ptr()), None, None, None) == INVALID
    assert L.moe_router_topk(ctypes.byref(r), v(x.data_ptr()), 0, 8, v(idx.data_ptr()),
                             v(wt.data_ptr()), None, None, None) == INVALID
    r256, k2 = mat(256, 256, bits=8)
    assert L.moe_router_topk(ctypes.byref(r256), v(x.data_ptr()), 1, 8, v(idx.data_ptr()),
                             v(wt.data_ptr()), None, None, None) == UNSUP
    # expert layer: workspace too small, wrong matrix shapes
    H, I, E = 128, 64, 16
    mats = {n: mat(*(rc), bits=4) for n, rc in (("gate", (I, H)), ("up", (I, H)),
                                                ("down", (H, I)), ("sh_gate", (I, H)),
                                                ("sh_up", (I, H)), ("sh_down", (H, I)))}
    lay = qmoe.CMoeLayer(*(mats[n][0] for n in ("gate", "up", "down", "sh_gate", "sh_up",
                                                 "sh_down")), E, H, I)
    need = L.moe_expert_workspace_bytes(ctypes.byref(lay), 8)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y = torch.zeros(H, dtype=torch.float16, device="cuda")
    xx = torch.zeros(H, dtype=torch.float16, device="cuda")
    args = lambda n: (ctypes.byref(lay), v(xx.data_ptr()), v(idx.data_ptr()), v(wt.data_ptr()), 8,
                      v(y.data_ptr()), v(ws.data_ptr()), n, None, None)
    assert L.moe_expert_qmlp(*args(need)) == 0
    assert L.moe_expert_qmlp(*args(need - 1)) == WS
    lay.down.rows = 64
    assert L.moe_expert_qmlp(*args(need)) == INVALID
    torch.cuda.synchronize()
    assert qmoe.qmoe_check_status() == 0
