"""Host-memory expert streaming through the LFU cache (moe_cache_layer) on
the GPU: every token's output against the oracle's layer, the router's ids
against the oracle's selection, and the cache's hits, misses and slot
contents against the oracle's LFU plan replayed on the same ids."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, f16_bits

pytestmark = pytest.mark.gpu


def stream_tokens(m, E, H, I, nslots, k, x16):
    layer = qmoe.ExpertCacheLayer(m, E, H, I, nslots=nslots)
    ref_plan = oracle.LfuCache(nslots)
    L = oracle.Layer(m, E, H, I)
    idx = torch.empty(k, dtype=torch.int32, device="cuda")
    wt = torch.empty(k, dtype=torch.float32, device="cuda")
    hits = misses = 0
    for t in range(x16.shape[0]):
        x = torch.from_numpy(x16[t].view(np.float16).copy()).cuda()
        y = layer.forward(x, top_k=k, idx=idx, weights=wt)
        assert qmoe.qmoe_check_status() == 0
        ids = idx.cpu().numpy()
        _, oidx, _ = oracle.router(*m["router"], E, H, 8, x16[t:t + 1], k)
        assert np.array_equal(ids, oidx[0]), "token %d: router ids" % t
        y64, _ = L.moe(x16[t:t + 1], ids[None], wt.cpu().numpy()[None].astype(np.float64))
        assert_close(f16_bits(y).view(np.float16), y64[0], what="token %d" % t)
        _, miss = ref_plan.step(ids)
        misses += len(miss)
        hits += k - len(miss)
    h, mi, nbytes, slots = layer.stats()
    assert (h, mi) == (hits, misses)
    assert slots.tolist() == ref_plan.expert.tolist()
    per_expert = sum(int(np.prod(m[n][0].shape[1:])) * 4 + 2 * int(np.prod(m[n][1].shape[1:])) * 2
                     for n in ("gate", "up", "down"))
    assert nbytes == misses * per_expert
    return hits, misses


@pytest.mark.parametrize("rho", [0.0, 0.95])
def test_small_layer_token_stream(cuda_dev, rho):
    E, H, I, k = 32, 512, 256, 8
    m = synth.moe_layer(21, 0, E=E, H=H, I=I)
    x16 = synth.correlated_tokens(21, 24, H, rho)
    hits, misses = stream_tokens(m, E, H, I, 16, k, x16)
    assert misses >= k   # the cache starts empty


@pytest.mark.slow
def test_moe_e128_layer_token_stream(cuda_dev):
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK
    m = synth.moe_layer(22, 0)
    x16 = synth.correlated_tokens(22, 10, H, 0.9)
    stream_tokens(m, E, H, I, 16, k, x16)
