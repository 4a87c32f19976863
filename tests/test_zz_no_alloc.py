"""moe_expert_qmlp_noalloc: the decode MoE layer for callers that cannot
allocate device memory (its scratch is built into the library).  Called
through the C ABI and checked against the CPU oracle and against
moe_expert_qmlp, the entry point that takes a caller-owned workspace, on two
calls in a row; after a call of another shape has left data where this
shape's counters live; and a rejected call must put nothing on its stream.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = qmoe.lib().moe_expert_qmlp_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _call_noalloc(G, x, idx, wt, y):
    return _noalloc_fn()(ctypes.byref(G.c), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
              ctypes.c_void_p(wt.data_ptr()), idx.numel(), ctypes.c_void_p(y.data_ptr()), None,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _layer_case(seed, E, H, I, k):
    m = synth.moe_layer(seed, 0, E=E, H=H, I=I)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    x16 = synth.activations(seed, 1, H)
    _, idx, wt = oracle.router(*m["router"], E, H, 8, x16, k)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt)
    x = torch.from_numpy(x16.view(np.float16).copy()).cuda().reshape(-1)
    idx_d = torch.from_numpy(idx[0].astype(np.int32)).cuda()
    wt_d = torch.from_numpy(wt[0].astype(np.float32)).cuda()
    return G, x, idx_d, wt_d, y64[0]


def _noalloc_y(G, x, idx_d, wt_d, H):
    y = torch.full((H,), float("nan"), dtype=torch.float16, device="cuda")
    assert _call_noalloc(G, x, idx_d, wt_d, y) == 0
    assert qmoe.qmoe_check_status() == 0
    return f16_bits(y).view(np.float16).astype(np.float64)


def test_noalloc_matches_workspace_entry_point(cuda_dev):
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    G, x, idx_d, wt_d, y64 = _layer_case(21, E, H, I, 8)
    ref = f16_bits(qmoe.moe_expert_qmlp(G, x, idx_d, wt_d)).view(np.float16).astype(np.float64)
    assert qmoe.qmoe_check_status() == 0
    assert_close(ref, y64, what="workspace entry point vs oracle")
    for _ in range(2):
        y = _noalloc_y(G, x, idx_d, wt_d, H)
        assert_close(y, ref, what="no-alloc vs workspace entry point")
        assert_close(y, y64, what="no-alloc vs oracle")


def test_noalloc_clears_counters_left_dirty_by_another_shape(cuda_dev):
    """The scratch keeps the last call's contents.  A call of the full decode
    shape writes its fp32 intermediates over the bytes where a smaller shape
    keeps its arrival counters; the smaller call must clear them and still
    match the oracle (and so must the big shape after it)."""
    big = _layer_case(22, synth.MOE_E, synth.MOE_H, synth.MOE_I, 8)
    small = _layer_case(23, 32, 512, 256, 2)
    lib = qmoe.lib()
    # the small shape's counters lie inside the region the big shape writes
    small_ws = lib.moe_expert_workspace_bytes(ctypes.byref(small[0].c), 2)
    counters_off = small_ws - 256   # the counters are the layout's last 256-byte block
    assert counters_off < 9 * synth.MOE_I * 4   # inside the big shape's h region
    for case, H in ((big, synth.MOE_H), (small, 512), (big, synth.MOE_H), (small, 512)):
        G, x, idx_d, wt_d, y64 = case
        assert_close(_noalloc_y(G, x, idx_d, wt_d, H), y64, what="no-alloc after another shape")


def test_noalloc_rejected_call_enqueues_nothing(cuda_dev):
    """A call that fails its argument checks returns before it puts anything
    on its stream (so it cannot clear the counters of a call in flight).  The
    stream is put in capture mode only to count what the call enqueued."""
    from cuda.bindings import runtime as rt
    E, H, I = 32, 512, 256
    G, x, idx_d, wt_d, _ = _layer_case(24, E, H, I, 2)
    y = torch.empty(H, dtype=torch.float16, device="cuda")
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    fn = _noalloc_fn()
    bad = [
        (x.data_ptr(), 0),                 # top_k out of range
        (x.data_ptr(), E + 1),
        (x.data_ptr() + 1, 2),             # x not 2-byte aligned
    ]
    for xp, k in bad:
        err, = rt.cudaStreamBeginCapture(s.cuda_stream,
                                        rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
        assert err == rt.cudaError_t.cudaSuccess
        rc = fn(ctypes.byref(G.c), ctypes.c_void_p(xp), ctypes.c_void_p(idx_d.data_ptr()),
                ctypes.c_void_p(wt_d.data_ptr()), k, ctypes.c_void_p(y.data_ptr()), None,
                ctypes.c_void_p(s.cuda_stream))
        err, graph = rt.cudaStreamEndCapture(s.cuda_stream)
        assert err == rt.cudaError_t.cudaSuccess
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        rt.cudaGraphDestroy(graph)
        assert rc != 0, "the call should have been rejected"
        assert n == 0, "a rejected call enqueued %d operation(s)" % n


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
