"""Expert-parallel MoE layer (moe_expert_qmlp_ep) on one GPU: every rank's
share is computed in turn, each from a layer holding only that rank's
experts, and the shares must add up to the whole layer (the oracle's, and the
single-GPU kernel's).  No rank waits for another, so one device can play all
of them; the all-reduce itself is covered on CPU (test_dist_ep.py)."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import REL_TOL, assert_close, f16_bits

pytestmark = pytest.mark.gpu


def ep_shares(m, E, H, I, k, world, x16):
    x = torch.from_numpy(x16.view(np.float16).copy()).cuda().reshape(-1)
    G0 = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt, _ = qmoe.moe_router_topk(G0.router, x.reshape(1, -1), k)
    parts = []
    for r in range(world):
        Gr = qmoe.MoELayer.from_numpy(m, E, H, I, rank=r, world=world)
        parts.append(qmoe.moe_expert_qmlp_ep(Gr, x, idx.reshape(-1), wt.reshape(-1), r, world)
                     .cpu().numpy().astype(np.float64))
    assert qmoe.qmoe_check_status() == 0
    y1 = f16_bits(qmoe.moe_expert_qmlp(G0, x, idx.reshape(-1), wt.reshape(-1)))
    return parts, idx.cpu().numpy(), wt.cpu().numpy(), y1


@pytest.mark.parametrize("E,H,I,k", [(32, 512, 256, 8), (16, 1024, 128, 4)])
@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_shares_add_up_to_the_layer(cuda_dev, E, H, I, k, world):
    m = synth.moe_layer(11, 0, E=E, H=H, I=I)
    x16 = synth.activations(11 + world, 1, H)
    parts, idx, wt, y1 = ep_shares(m, E, H, I, k, world, x16)
    _, oidx, owt = oracle.router(*m["router"], E, H, 8, x16, k)
    assert np.array_equal(idx, oidx)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    total = np.sum(parts, axis=0)
    assert_close(total, y64[0], what="sum of %d shares" % world)
    assert_close(total, y1.view(np.float16).astype(np.float64), what="vs single GPU")
    for r in range(world):
        held = [j for j in range(k) if qmoe.expert_owner(int(idx[0, j]), E, world) == r]
        if r > 0 and not held:
            assert not parts[r].any(), "rank %d holds no chosen expert: zeros" % r


@pytest.mark.slow
def test_e128_layer_eight_ranks(cuda_dev):
    """The 128-expert, H=2816, I=704 decode layer over 8 ranks of 16 experts."""
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK
    m = synth.moe_layer(0, 5)
    x16 = synth.activations(0, 1, H, layer=5)
    parts, idx, wt, y1 = ep_shares(m, E, H, I, k, 8, x16)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    assert_close(np.sum(parts, axis=0), y64[0], what="E128 over 8 ranks")


def test_rank_without_experts_and_conversion(cuda_dev):
    """world = E: each rank holds one expert, most hold none of the chosen
    ones and return zeros; the fp32 -> fp16 kernel rounds like numpy."""
    E, H, I, k = 16, 256, 64, 4
    m = synth.moe_layer(5, 0, E=E, H=H, I=I)
    x16 = synth.activations(5, 1, H)
    parts, idx, wt, _ = ep_shares(m, E, H, I, k, E, x16)
    chosen = set(int(e) for e in idx[0])
    for r in range(1, E):
        if r not in chosen:
            assert not parts[r].any()
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    assert_close(np.sum(parts, axis=0), y64[0], what="one expert per rank")
    v = torch.randn(10001, dtype=torch.float32, device="cuda") * 1000
    v[:4] = torch.tensor([65504.0, 65520.0, -70000.0, 1e-8])
    got = f16_bits(qmoe.f32_to_f16(v))
    want = v.cpu().numpy().astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_ep_argument_errors(cuda_dev):
    import ctypes
    E, H, I, k = 16, 256, 64, 4
    m = synth.moe_layer(5, 0, E=E, H=H, I=I)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    x = torch.zeros(H, dtype=torch.float16, device="cuda")
    idx = torch.zeros(k, dtype=torch.int32, device="cuda")
    wt = torch.zeros(k, dtype=torch.float32, device="cuda")
    y = torch.zeros(H, dtype=torch.float32, device="cuda")
    ws = qmoe.expert_workspace(G, k)
    call = lambda rank, world, yp: qmoe.lib().moe_expert_qmlp_ep(
        ctypes.byref(G.c), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(wt.data_ptr()), k, rank, world, ctypes.c_void_p(yp), ctypes.c_void_p(ws.data_ptr()),
        ws.numel(), None, None)
    assert call(0, 1, y.data_ptr()) == 0
    assert call(0, 3, y.data_ptr()) == -1        # world does not divide E
    assert call(2, 2, y.data_ptr()) == -1        # rank out of range
    assert call(0, 0, y.data_ptr()) == -1
    assert call(0, 2, None) == -1
    assert call(0, 2, y.data_ptr() + 2) == -2    # fp32 alignment
    torch.cuda.synchronize()
