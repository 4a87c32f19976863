"""moe_router_topk on the GPU against the CPU oracle.

Index parity is bit-exact in this sense: the oracle's selection applied to the
GPU's own fp32 logits reproduces the GPU's indices exactly, and the GPU's
indices equal the oracle's fp64 selection except where the k-th and (k+1)-th
logits are closer than the fp32 rounding of the logits (counted; none at these
sizes)."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, to_dev_f16

pytestmark = pytest.mark.gpu


def route(P, S, B, E, K, bits, x16, k):
    R = qmoe.QMatrix.from_numpy(P, S, B, E, K, bits)
    idx, wt, lg = qmoe.moe_router_topk(R, to_dev_f16(x16), k, want_logits=True)
    assert qmoe.qmoe_check_status() == 0
    return idx.cpu().numpy(), wt.cpu().numpy(), lg.cpu().numpy()


def check_against_oracle(P, S, B, E, K, bits, x16, k):
    idx, wt, lg = route(P, S, B, E, K, bits, x16, k)
    l64, oidx, owt = oracle.router(P, S, B, E, K, bits, x16, k)
    # logits: normwise
    assert np.abs(lg - l64).max() <= 1e-5 * np.abs(l64).max()
    # selection on the GPU's own logits is reproduced exactly
    sidx, swt = oracle.topk_from_logits(lg, k)
    assert np.array_equal(idx, sidx)
    assert_close(wt, swt, what="weights vs selection on device logits")
    # against the fp64 selection: equal except at genuine near-ties
    srt = -np.sort(-l64, axis=1)
    near = np.zeros(len(x16), bool)
    if k < E:
        near = (srt[:, k - 1] - srt[:, k]) < 1e-5 * np.abs(l64).max()
    diff = np.any(idx != oidx, axis=1)
    assert not np.any(diff & ~near), "index mismatch away from a near-tie"
    same = ~diff
    if same.any():
        assert_close(wt[same], owt[same], what="weights vs oracle")
    np.testing.assert_allclose(wt.sum(axis=1), 1.0, rtol=1e-5)
    return int(near.sum())


@pytest.mark.parametrize("T", [1, 2, 4, 8, 16, 32, 64, 128])
def test_router_e128_k2816(cuda_dev, T):
    E, K = 128, 2816
    P, S, B = synth.router(2, E, K)
    x16 = synth.activations(20 + T, T, K)
    assert check_against_oracle(P, S, B, E, K, 8, x16, 8) == 0


@pytest.mark.parametrize("E,K,k", [(8, 64, 1), (16, 128, 4), (24, 192, 8), (40, 704, 16),
                                   (128, 2816, 1), (128, 2816, 16), (64, 1024, 8)])
@pytest.mark.parametrize("bits", [8, 4])
def test_router_shapes(cuda_dev, E, K, k, bits):
    P, S, B = synth.qmatrix(synth.rng(E, K, k), E, K, bits, synth.ROUTER_SCALE, synth.ROUTER_BIAS)
    x16 = synth.activations(E + K, 11, K)
    check_against_oracle(P, S, B, E, K, bits, x16, k)


def test_zero_input_ties_lowest_index(cuda_dev):
    E, K = 128, 2816
    P, S, B = synth.router(3, E, K)
    idx, wt, lg = route(P, S, B, E, K, 8, np.zeros((3, K), np.uint16), 8)
    assert np.all(lg == 0)
    assert np.all(idx == np.arange(8)[None, :])
    assert np.all(wt == 0.125)


def test_duplicate_rows_tie(cuda_dev):
    """Two identical router rows give bit-identical logits; the lower index
    must come first."""
    E, K = 128, 2816
    P, S, B = synth.router(4, E, K)
    P, S, B = P.copy(), S.copy(), B.copy()
    B[[5, 9, 77], :] = synth.to_f16_bits(np.full(K // 64, 10.0))
    for r in (9, 77):
        P[r], S[r], B[r] = P[5], S[5], B[5]
    x16 = synth.to_f16_bits(np.abs(synth.activations(4, 2, K).view(np.float16)).astype(np.float64))
    idx, wt, lg = route(P, S, B, E, K, 8, x16, 8)
    assert np.all(lg[:, 5] == lg[:, 9]) and np.all(lg[:, 5] == lg[:, 77])
    assert np.all(idx[:, :3] == [5, 9, 77])
    assert np.all(wt[:, 0] == wt[:, 1])
