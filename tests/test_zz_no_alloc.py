"""moe_expert_qmlp_noalloc: the decode MoE layer for callers that cannot
allocate device memory (its scratch is built into the library).  Called
through the C ABI and checked against moe_expert_qmlp, the entry point that
takes a caller-owned workspace, on two calls in a row.  This file is collected
last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits

pytestmark = pytest.mark.gpu


def _call_noalloc(G, x, idx, wt, y):
    lib = qmoe.lib()
    fn = lib.moe_expert_qmlp_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(ctypes.byref(G.c), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
              ctypes.c_void_p(wt.data_ptr()), idx.numel(), ctypes.c_void_p(y.data_ptr()), None,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point(cuda_dev):
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    m = synth.moe_layer(21, 0)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    x16 = synth.activations(21, 1, H)
    _, idx, wt = oracle.router(*m["router"], E, H, 8, x16, 8)
    x = torch.from_numpy(x16.view(np.float16).copy()).cuda().reshape(-1)
    idx_d = torch.from_numpy(idx[0].astype(np.int32)).cuda()
    wt_d = torch.from_numpy(wt[0].astype(np.float32)).cuda()
    ref = f16_bits(qmoe.moe_expert_qmlp(G, x, idx_d, wt_d)).view(np.float16).astype(np.float64)
    assert qmoe.qmoe_check_status() == 0
    for _ in range(2):
        y = torch.full((H,), float("nan"), dtype=torch.float16, device="cuda")
        assert _call_noalloc(G, x, idx_d, wt_d, y) == 0
        assert qmoe.qmoe_check_status() == 0
        assert_close(f16_bits(y).view(np.float16), ref, what="no-alloc vs workspace entry point")


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_dev):
    """A layer whose workspace would exceed the built-in 1 MiB is refused
    before anything is enqueued (QMOE_ERR_WORKSPACE)."""
    H, I, E = 16384, 8192, 16
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")   # never read: rejected first
    p = buf.data_ptr()
    mk = lambda r, c: qmoe.CQMatrix(p, p, p, r, c, 4, 64)
    lay = qmoe.CMoeLayer(mk(I, H), mk(I, H), mk(H, I), mk(I, H), mk(I, H), mk(H, I), E, H, I)
    lib = qmoe.lib()
    assert lib.moe_expert_workspace_bytes(ctypes.byref(lay), 16) > (1 << 20)
    fn = lib.moe_expert_qmlp_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    rc = fn(ctypes.byref(lay), ctypes.c_void_p(p), ctypes.c_void_p(p), ctypes.c_void_p(p), 16,
            ctypes.c_void_p(p), None, None)
    assert rc == -7
