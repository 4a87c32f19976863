"""The tensor-core (tcgen05) path of the prefill chunk: experts with many
tokens (and the shared expert) as a matrix product on the tensor cores,
checked token by token against the CPU oracle, alone and next to the
streaming kernels that take the other experts."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits

pytestmark = pytest.mark.gpu


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=dtype)).cuda()


@pytest.fixture
def tensor_min():
    """Set the token threshold of the tensor-core path for one test."""
    old = []

    def set_(n):
        old.append(qmoe.qmoe_set_prefill_tensor_min(n))
    yield set_
    if old:
        qmoe.qmoe_set_prefill_tensor_min(old[0])


def run_chunk(G, x16, idx, wt):
    y = qmoe.moe_prefill_qgemm(G, dev(x16.view(np.float16), np.float16), dev(idx, np.int32),
                               dev(wt, np.float32))
    flags = qmoe.qmoe_check_status()
    return f16_bits(y).view(np.float16), flags


def check_tokens(y, y64, what):
    assert_close(y, y64, what=what)
    for t in range(y.shape[0]):
        assert_close(y[t], y64[t], what="%s, token %d" % (what, t))


@pytest.mark.parametrize("E,H,I,T,k,tmin", [(16, 256, 128, 33, 8, 16), (32, 512, 192, 128, 8, 16),
                                            (64, 1024, 256, 100, 16, 16), (16, 256, 64, 40, 4, 1),
                                            (8, 512, 320, 128, 4, 16)])
def test_chunks_with_tensor_core_slots(cuda_dev, tensor_min, E, H, I, T, k, tmin):
    tensor_min(tmin)
    m = synth.moe_layer(E + T + 3, 0, E=E, H=H, I=I, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(E + T + 3, T=T, E=E, k=k)
    x16 = synth.activations(E + T + 3, T, H)
    y, flags = run_chunk(G, x16, idx, wt)
    assert flags == 0
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    check_tokens(y, y64, "tensor-core chunk %s" % ((E, H, I, T, k, tmin),))


def test_same_result_either_path(cuda_dev, tensor_min):
    """The two paths agree with each other within the tolerance (and with the
    oracle) on the same chunk."""
    E, H, I, T, k = 32, 512, 256, 64, 8
    m = synth.moe_layer(41, 0, E=E, H=H, I=I, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(41, T=T, E=E, k=k)
    x16 = synth.activations(41, T, H)
    tensor_min(0)
    y0, f0 = run_chunk(G, x16, idx, wt)
    qmoe.qmoe_set_prefill_tensor_min(1)
    y1, f1 = run_chunk(G, x16, idx, wt)
    assert f0 == 0 and f1 == 0
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    check_tokens(y0, y64, "streaming path")
    check_tokens(y1, y64, "tensor-core path")


@pytest.mark.slow
def test_chunk128_zipf_every_token(cuda_dev, tensor_min):
    """The 128-token Zipf(1.1) chunk of the 128-expert layer with the default
    threshold (16 tokens): every token against the oracle."""
    tensor_min(qmoe.TENSOR_MIN_DEFAULT)
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    m = synth.moe_layer(4, 0)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(4)
    x16 = synth.activations(4, synth.PREFILL_T, H)
    y, flags = run_chunk(G, x16, idx, wt)
    assert flags == 0
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    check_tokens(y, y64, "128-token chunk, tensor-core path")


@pytest.mark.slow
def test_dense_routing_every_slot_full(cuda_dev, tensor_min):
    """Every token routed to experts 0..7: nine slots of 128 tokens each, all
    on the tensor cores (the dense case); a sample of tokens against the
    oracle."""
    tensor_min(qmoe.TENSOR_MIN_DEFAULT)
    E, H, I, T, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, 128, 8
    m = synth.moe_layer(6, 0)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    _, wt = synth.zipf_routing(6, T=T, E=E, k=k)
    x16 = synth.activations(6, T, H)
    y, flags = run_chunk(G, x16, idx, wt)
    assert flags == 0
    rows = np.arange(0, T, 9)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16[rows], idx[rows], wt[rows].astype(np.float64))
    check_tokens(y[rows], y64, "dense routing")


def test_bad_expert_ids_with_tensor_cores(cuda_dev, tensor_min):
    tensor_min(1)
    E, H, I, T, k = 16, 256, 64, 24, 4
    m = synth.moe_layer(78, 0, E=E, H=H, I=I, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(78, T=T, E=E, k=k)
    idx = idx.copy()
    idx[2, 1] = 99
    idx[5, 0] = -3
    x16 = synth.activations(78, T, H)
    y, flags = run_chunk(G, x16, idx, wt)
    assert flags & qmoe.DEV_BAD_EXPERT
    keep = (idx >= 0) & (idx < E)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, np.where(keep, idx, 0).astype(np.int32),
                                          np.where(keep, wt, 0.0).astype(np.float64))
    check_tokens(y, y64, "bad ids dropped")
