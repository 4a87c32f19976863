"""Prefill chunk through the MoE layer (moe_prefill_qgemm) and the grouping
(moe_group_tokens) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits

pytestmark = pytest.mark.gpu


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=dtype)).cuda()


@pytest.mark.parametrize("T,k,E", [(128, 8, 128), (1, 8, 128), (37, 3, 16), (128, 16, 256),
                                   (5, 1, 8)])
def test_grouping_bit_exact(cuda_dev, T, k, E):
    g = np.random.default_rng(T * k + E)
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, pairs = qmoe.moe_group_tokens(dev(idx, np.int32), E)
    oc, oo, op = oracle.group(idx, E)
    assert np.array_equal(counts.cpu().numpy(), oc)
    assert np.array_equal(offsets.cpu().numpy(), oo)
    assert np.array_equal(pairs.cpu().numpy(), op)


def test_grouping_zipf_chunk(cuda_dev):
    idx, _ = synth.zipf_routing(0)
    counts, offsets, pairs = qmoe.moe_group_tokens(dev(idx, np.int32), 128)
    oc, oo, op = oracle.group(idx, 128)
    assert np.array_equal(counts.cpu().numpy(), oc) and np.array_equal(pairs.cpu().numpy(), op)


def run_prefill(G, x16, idx, wt):
    y = qmoe.moe_prefill_qgemm(G, dev(x16.view(np.float16), np.float16), dev(idx, np.int32),
                               dev(wt, np.float32))
    flags = qmoe.qmoe_check_status()
    return f16_bits(y), flags


@pytest.mark.parametrize("E,H,I,T,k", [(16, 256, 64, 7, 4), (16, 256, 128, 33, 8),
                                       (32, 512, 192, 128, 8), (8, 256, 64, 1, 1),
                                       (64, 1024, 256, 100, 16)])
def test_small_chunks_full_compare(cuda_dev, E, H, I, T, k):
    m = synth.moe_layer(E + T, 0, E=E, H=H, I=I, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(E + T, T=T, E=E, k=k)
    x16 = synth.activations(E + T, T, H)
    y, flags = run_prefill(G, x16, idx, wt)
    assert flags == 0
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    assert_close(y.view(np.float16), y64, what="prefill %s" % ((E, H, I, T, k),))
    for t in range(T):   # each token on its own scale
        assert_close(y.view(np.float16)[t], y64[t], what="prefill %s token %d" % ((E, H, I, T, k), t))


@pytest.fixture(scope="module")
def chunk128():
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    m = synth.moe_layer(4, 0)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(4)
    x16 = synth.activations(4, synth.PREFILL_T, H)
    return m, G, idx, wt, x16


@pytest.mark.slow
def test_chunk128_every_token(cuda_dev, chunk128):
    """The 128-token chunk with Zipf(1.1) routing: every output of every token
    against the oracle, each token on its own scale (and the chunk as a
    whole)."""
    m, G, idx, wt, x16 = chunk128
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    y, flags = run_prefill(G, x16, idx, wt)
    assert flags == 0
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx, wt.astype(np.float64))
    yv = y.view(np.float16)
    assert_close(yv, y64, what="128-token chunk")
    for t in range(synth.PREFILL_T):
        assert_close(yv[t], y64[t], what="128-token chunk, token %d" % t)


def test_decode_layer_on_chunk_tokens_matches_oracle(cuda_dev, chunk128):
    """The per-token decode layer (moe_expert_qmlp) on tokens of the chunk,
    with the chunk's routing, against the oracle."""
    m, G, idx, wt, x16 = chunk128
    E, H, I = synth.MOE_E, synth.MOE_H, synth.MOE_I
    L = oracle.Layer(m, E, H, I)
    for t in (0, 63, 127):
        yd = qmoe.moe_expert_qmlp(G, dev(x16[t].view(np.float16), np.float16), dev(idx[t], np.int32),
                                  dev(wt[t], np.float32))
        assert qmoe.qmoe_check_status() == 0
        y64, _ = L.moe(x16[t:t + 1], idx[t:t + 1], wt[t:t + 1].astype(np.float64))
        assert_close(f16_bits(yd).view(np.float16), y64[0], what="decode layer, token %d" % t)


def test_bad_expert_ids_flagged(cuda_dev):
    E, H, I, T, k = 16, 256, 64, 9, 4
    m = synth.moe_layer(77, 0, E=E, H=H, I=I, with_router=False)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    idx, wt = synth.zipf_routing(77, T=T, E=E, k=k)
    idx = idx.copy()
    idx[2, 1] = 99
    idx[5, 0] = -3
    x16 = synth.activations(77, T, H)
    y, flags = run_prefill(G, x16, idx, wt)
    assert flags & qmoe.DEV_BAD_EXPERT
    keep = (idx >= 0) & (idx < E)
    wt2 = np.where(keep, wt, 0.0)
    idx2 = np.where(keep, idx, 0).astype(np.int32)
    y64, _ = oracle.Layer(m, E, H, I).moe(x16, idx2, wt2.astype(np.float64))
    assert_close(y.view(np.float16), y64, what="bad ids dropped")


def test_repeat_calls_bitwise_identical(cuda_dev, chunk128):
    m, G, idx, wt, x16 = chunk128
    a, _ = run_prefill(G, x16, idx, wt)
    b, _ = run_prefill(G, x16, idx, wt)
    assert np.array_equal(a, b)
