"""Decode MoE layer (moe_expert_qmlp) on the GPU against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits, to_dev_f16

pytestmark = pytest.mark.gpu

E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I


@pytest.fixture(scope="module")
def layer_full():
    m = synth.moe_layer(7, 0)
    return m, qmoe.MoELayer.from_numpy(m, E, H, I), oracle.Layer(m, E, H, I)


def gpu_layer(G, x16, idx, wt, ws=None):
    y = qmoe.moe_expert_qmlp(G, to_dev_f16(x16).reshape(-1),
                             torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda(),
                             torch.from_numpy(np.ascontiguousarray(wt, np.float32)).cuda(),
                             workspace=ws)
    return y


def test_moe_layer_e128_oracle_routing(cuda_dev, layer_full):
    """Full-size layer; routing from the oracle's router (fp64), weights passed
    to both sides as the same fp32 values."""
    m, G, L = layer_full
    x16 = synth.activations(7, 1, H)
    _, idx, wt = oracle.router(*m["router"], E, H, 8, x16, 8)
    wt32 = wt.astype(np.float32)
    y = gpu_layer(G, x16, idx[0], wt32[0])
    assert qmoe.qmoe_check_status() == 0
    y64, _ = L.moe(x16, idx, wt32.astype(np.float64))
    assert_close(f16_bits(y).view(np.float16), y64[0], what="E128 H2816 I704 layer")


def test_moe_layer_e128_router_then_experts(cuda_dev, layer_full):
    """The device path end to end: GPU router ids feed the GPU experts."""
    m, G, L = layer_full
    for seed in range(3):
        x16 = synth.activations(100 + seed, 1, H)
        xd = to_dev_f16(x16)
        idx, wt, _ = qmoe.moe_router_topk(G.router, xd, 8)
        y = qmoe.moe_expert_qmlp(G, xd.reshape(-1), idx.reshape(-1), wt.reshape(-1))
        assert qmoe.qmoe_check_status() == 0
        _, oidx, _ = oracle.router(*m["router"], E, H, 8, x16, 8)
        assert np.array_equal(idx.cpu().numpy(), oidx)
        y64, _ = L.moe(x16, idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64))
        assert_close(f16_bits(y).view(np.float16), y64[0], what="router->experts")


def test_workspace_reuse_deterministic(cuda_dev, layer_full):
    m, G, L = layer_full
    ws = qmoe.expert_workspace(G, 8)
    x16 = synth.activations(8, 1, H)
    idx = np.array([3, 120, 7, 64, 0, 127, 55, 9], np.int32)
    wt = np.full(8, 0.125, np.float32)
    first = f16_bits(gpu_layer(G, x16, idx, wt, ws)).copy()
    for _ in range(4):
        assert np.array_equal(f16_bits(gpu_layer(G, x16, idx, wt, ws)), first)
    assert torch.count_nonzero(ws[-(H // 16) * 4:]) == 0   # counters back to zero


def test_zero_input_zero_output(cuda_dev, layer_full):
    m, G, L = layer_full
    y = gpu_layer(G, np.zeros((1, H), np.uint16), np.arange(8, dtype=np.int32),
                  np.full(8, 0.125, np.float32))
    assert np.all(f16_bits(y) == 0)


def test_bad_expert_id_flagged_and_skipped(cuda_dev, layer_full):
    m, G, L = layer_full
    x16 = synth.activations(9, 1, H)
    idx = np.array([3, 200, 7, -1, 0, 127, 55, 9], np.int32)
    wt = np.full(8, 0.125, np.float32)
    y = gpu_layer(G, x16, idx, wt)
    flags = qmoe.qmoe_check_status()
    assert flags & qmoe.DEV_BAD_EXPERT
    keep = (idx >= 0) & (idx < E)
    y64, _ = L.moe(x16, idx[keep][None], wt[keep][None].astype(np.float64))
    assert_close(f16_bits(y).view(np.float16), y64[0], what="bad ids skipped")


@pytest.mark.parametrize("k", [1, 2, 8, 16])
def test_small_layer_topk(cuda_dev, k):
    e, h, i = 16, 128, 64
    m = synth.moe_layer(30 + k, 0, E=e, H=h, I=i, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, e, h, i)
    L = oracle.Layer(m, e, h, i)
    g = np.random.default_rng(k)
    idx = g.permutation(e)[:k].astype(np.int32)
    wt = g.uniform(0.1, 1, k).astype(np.float32)
    wt /= wt.sum()
    x16 = synth.activations(31 + k, 1, h)
    y = gpu_layer(G, x16, idx, wt)
    assert qmoe.qmoe_check_status() == 0
    y64, _ = L.moe(x16, idx[None], wt[None].astype(np.float64))
    assert_close(f16_bits(y).view(np.float16), y64[0], what="small k=%d" % k)


def test_other_shapes(cuda_dev):
    for (e, h, i) in ((8, 256, 192), (32, 1024, 512), (128, 2048, 1408)):
        m = synth.moe_layer(40 + h, 0, E=e, H=h, I=i, with_router=False)
        G = qmoe.MoELayer.from_numpy(m, e, h, i)
        L = oracle.Layer(m, e, h, i)
        idx = np.arange(min(8, e), dtype=np.int32)[::-1].copy()
        wt = np.linspace(0.3, 0.05, len(idx)).astype(np.float32)
        x16 = synth.activations(41 + h, 1, h)
        y = gpu_layer(G, x16, idx, wt)
        assert qmoe.qmoe_check_status() == 0
        y64, _ = L.moe(x16, idx[None], wt[None].astype(np.float64))
        assert_close(f16_bits(y).view(np.float16), y64[0], what="shape %s" % ((e, h, i),))
