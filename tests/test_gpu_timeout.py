"""A device wait that cannot complete ends the launch with a timeout status
instead of hanging, and the context stays usable.

The fused decode's layer barrier waits until an arrival counter in its
workspace reaches (layers done) x (arrivals per layer).  The test presets that
counter to 2^32 - 1: after the first layer's arrivals it has wrapped to just
below the target of the second layer, so that wait can never complete (a
flag nothing sets).  With the wait limit lowered to 1 ms the launch must return, report
QMOE_DEV_TIMEOUT, and leave its control words at zero; after the workspace is
zeroed again, the same call gives the oracle's results."""
import numpy as np
import pytest
import torch

from moe_expert_gemv_b200 import qmoe, synth
from tests.test_gpu_decode import check_layers, make_stack, run

pytestmark = pytest.mark.gpu


def test_decode_layer_barrier_times_out_and_recovers(cuda_dev):
    E, H, I, k, n = 16, 256, 64, 4, 2
    ms, stack = make_stack(61, n, E, H, I, k)
    x16 = np.concatenate([synth.activations(61 + l, 1, H, layer=l) for l in range(n)])
    xd = torch.from_numpy(x16.view(np.float16).copy()).cuda()
    old = qmoe.qmoe_set_decode_wait_limit_ns(1_000_000)
    try:
        ctl = stack.workspace[:4].view(torch.int32)
        ctl[0] = -1   # the layer arrival counter at 2^32 - 1
        torch.cuda.synchronize()
        qmoe.moe_decode_layers(stack, xd)
        flags = qmoe.qmoe_check_status()   # returns: the launch ended
        assert flags & qmoe.DEV_TIMEOUT
        # the last CTA out reset the control words
        assert torch.count_nonzero(stack.workspace[:16]) == 0
    finally:
        qmoe.qmoe_set_decode_wait_limit_ns(old)
    # the layer accumulators may hold partial sums: zero the workspace again
    stack.workspace.zero_()
    y, idx, wt, lg = run(stack, x16, E, k)
    check_layers(ms, E, H, I, k, x16, y, idx, wt, lg)
