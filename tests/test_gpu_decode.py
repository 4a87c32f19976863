"""Fused multi-layer decode (moe_decode_layers) against the CPU oracle: for
every layer the router's indices (bit-exact rules as in the router tests) and
the layer output y = shared(x) + sum_j wt_j expert_{idx_j}(x)."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import REL_TOL, assert_close, assert_close_f16, f16_bits

pytestmark = pytest.mark.gpu


def make_stack(seed, n, E, H, I, top_k):
    ms = [synth.moe_layer(seed, l, E=E, H=H, I=I) for l in range(n)]
    layers = [qmoe.MoELayer.from_numpy(m, E, H, I) for m in ms]
    return ms, qmoe.DecodeStack(layers, top_k)


def check_layers(ms, E, H, I, k, x16, y, idx, wt, lg, layers=None):
    for l in (range(len(ms)) if layers is None else layers):
        m = ms[l]
        l64, oidx, _ = oracle.router(*m["router"], E, H, 8, x16[l:l + 1], k)
        assert np.abs(lg[l] - l64[0]).max() <= 1e-5 * np.abs(l64).max()
        sidx, swt = oracle.topk_from_logits(lg[l:l + 1], k)
        assert np.array_equal(idx[l], sidx[0]), "layer %d: selection on device logits" % l
        assert_close(wt[l], swt[0], what="layer %d weights" % l)
        assert np.array_equal(idx[l], oidx[0]), "layer %d: indices differ from the fp64 oracle" % l
        y64, y16o = oracle.Layer(m, E, H, I).moe(x16[l:l + 1], idx[l:l + 1],
                                                 wt[l:l + 1].astype(np.float64))
        # (a layer whose outputs leave the fp16 range must give +-inf exactly
        # where the oracle's fp16 rounding does)
        assert_close_f16(y[l].view(np.float16), y64[0], y16o[0], what="layer %d output" % l)


def run(stack, x16, E, k):
    n = x16.shape[0]
    x = torch.from_numpy(x16.view(np.float16).copy()).cuda()
    idx = torch.empty(n, k, dtype=torch.int32, device="cuda")
    wt = torch.empty(n, k, dtype=torch.float32, device="cuda")
    lg = torch.empty(n, E, dtype=torch.float32, device="cuda")
    y = qmoe.moe_decode_layers(stack, x, idx=idx, weights=wt, logits=lg)
    assert qmoe.qmoe_check_status() == 0
    return f16_bits(y), idx.cpu().numpy(), wt.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("E,H,I,k,n", [(16, 256, 64, 4, 3), (32, 512, 128, 8, 2),
                                       (128, 1024, 256, 8, 2), (64, 768, 192, 16, 2),
                                       (8, 256, 64, 1, 4)])
def test_small_stacks(cuda_dev, E, H, I, k, n):
    ms, stack = make_stack(E + H, n, E, H, I, k)
    x16 = np.concatenate([synth.activations(7 + l, 1, H, layer=l) for l in range(n)])
    y, idx, wt, lg = run(stack, x16, E, k)
    check_layers(ms, E, H, I, k, x16, y, idx, wt, lg)


def test_router_ties_lowest_index(cuda_dev):
    """Exact ties inside the fused router: three identical router rows
    (experts 5, 9 and 77, made the largest; their logits come from different
    CTAs of a cluster) and an all-zero input (every logit 0) select the lower
    index first, as the oracle's rule does."""
    E, H, I, k = 128, 1024, 256, 8
    ms = [synth.moe_layer(11, l, E=E, H=H, I=I) for l in range(2)]
    P, S, B = (np.array(v, copy=True) for v in ms[0]["router"])
    B[[5, 9, 77], :] = synth.to_f16_bits(np.full(H // 64, 10.0))
    for r in (9, 77):
        P[r], S[r], B[r] = P[5], S[5], B[5]
    ms[0]["router"] = (P, S, B)
    stack = qmoe.DecodeStack([qmoe.MoELayer.from_numpy(m, E, H, I) for m in ms], k)
    xp = np.abs(synth.activations(12, 1, H, layer=0).view(np.float16)).astype(np.float64)
    x16 = np.concatenate([synth.to_f16_bits(xp), np.zeros((1, H), np.uint16)])
    y, idx, wt, lg = run(stack, x16, E, k)
    assert lg[0, 5] == lg[0, 9] == lg[0, 77]
    assert list(idx[0, :3]) == [5, 9, 77]
    assert np.all(lg[1] == 0) and list(idx[1]) == list(range(k)) and np.all(wt[1] == 1.0 / k)
    check_layers(ms, E, H, I, k, x16, y, idx, wt, lg)


def test_moe_e128_three_layers_and_repeat(cuda_dev):
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK
    ms, stack = make_stack(3, 3, E, H, I, k)
    x16 = np.concatenate([synth.activations(3, 1, H, layer=l) for l in range(3)])
    y, idx, wt, lg = run(stack, x16, E, k)
    check_layers(ms, E, H, I, k, x16, y, idx, wt, lg)
    # the workspace is back to zero; a second call reproduces the routing bit
    # for bit and the outputs within the tolerance (the cross-cluster fp32
    # sums of a layer output are atomic, so their order may change the last
    # bits)
    assert torch.count_nonzero(stack.workspace) == 0
    y2, idx2, wt2, lg2 = run(stack, x16, E, k)
    assert np.array_equal(idx, idx2) and np.array_equal(wt, wt2) and np.array_equal(lg, lg2)
    check_layers(ms, E, H, I, k, x16, y2, idx2, wt2, lg2)


def test_host_buffer_entry_point(cuda_dev):
    """moe_decode_layers_host: x from a pinned host buffer, y back into one,
    through the C call that enqueues both copies and the decode; outputs match
    the oracle like the device-buffer call."""
    E, H, I, k, n = 32, 512, 128, 8, 3
    ms, stack = make_stack(81, n, E, H, I, k)
    x16 = np.concatenate([synth.activations(81 + l, 1, H, layer=l) for l in range(n)])
    x_host = torch.from_numpy(x16.view(np.float16).copy()).pin_memory()
    y_host = torch.empty(n, H, dtype=torch.float16).pin_memory()
    x_dev = torch.empty(n, H, dtype=torch.float16, device="cuda")
    y_dev = torch.empty(n, H, dtype=torch.float16, device="cuda")
    qmoe.moe_decode_layers_host(stack, x_host, y_host, x_dev, y_dev)
    assert qmoe.qmoe_check_status() == 0   # synchronises the stream
    y, idx, wt, lg = run(stack, x16, E, k)
    assert_close(y_host.numpy(), y.view(np.float16).astype(np.float64), what="host entry vs device")
    for l in range(n):
        _, oidx, owt = oracle.router(*ms[l]["router"], E, H, 8, x16[l:l + 1], k)
        y64, _ = oracle.Layer(ms[l], E, H, I).moe(x16[l:l + 1], idx[l:l + 1],
                                                  wt[l:l + 1].astype(np.float64))
        assert_close(y_host.numpy()[l], y64[0], what="host entry layer %d vs oracle" % l)


def test_matches_unfused_path(cuda_dev):
    """Same bits as moe_router_topk + moe_expert_qmlp would give within the
    tolerance, and identical routing."""
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK
    ms, stack = make_stack(5, 2, E, H, I, k)
    x16 = np.concatenate([synth.activations(5, 1, H, layer=l) for l in range(2)])
    y, idx, wt, lg = run(stack, x16, E, k)
    for l in range(2):
        G = stack.layers[l]
        xd = torch.from_numpy(x16[l].view(np.float16).copy()).cuda()
        i2, w2, _ = qmoe.moe_router_topk(G.router, xd[None], k)
        y2 = qmoe.moe_expert_qmlp(G, xd, i2.reshape(-1), w2.reshape(-1))
        assert np.array_equal(i2.cpu().numpy()[0], idx[l])
        assert_close(y[l].view(np.float16), f16_bits(y2).view(np.float16).astype(np.float64),
                     what="fused vs unfused")


@pytest.mark.slow
def test_moe_e128_thirty_layers_all(cuda_dev):
    """The full decode step: 30 layers, 12.96 GB of weights, one launch.
    Every layer's routing and output is checked against the oracle; the host
    keeps only the routers while the stack is on the device and regenerates
    each layer from its seed for the oracle afterwards."""
    E, H, I, k, n = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK, synth.MOE_LAYERS
    layers, routers = [], []
    for l in range(n):
        m = synth.moe_layer(0, l)
        layers.append(qmoe.MoELayer.from_numpy(m, E, H, I))
        routers.append({"router": m["router"]})
        del m
    stack = qmoe.DecodeStack(layers, k)
    x16 = np.concatenate([synth.activations(0, 1, H, layer=l) for l in range(n)])
    y, idx, wt, lg = run(stack, x16, E, k)
    del stack, layers
    for l in range(n):
        m = synth.moe_layer(0, l)
        ms = [None] * n
        ms[l] = m
        check_layers(ms, E, H, I, k, x16, y, idx, wt, lg, layers=(l,))


def expected_pack(m, E, H, I):
    """The packed streaming layout, rebuilt with numpy from the row-major
    arrays (bytes): 8 router blocks of E/8 rows, then per expert (the shared
    expert last), per group g of 64 intermediate indices and per cluster rank
    r: gate rows 64g+8r..+7, the same up rows, and down rows H/8*r..+H/8-1
    restricted to inputs 64g..64g+63; codes of 16-byte chunk c of row i of a
    gate/up/router block at chunk (c & ~7) | ((c ^ i) & 7)."""
    GH, GI, Rr, Hc = H // 64, I // 64, E // 8, H // 8
    out = []
    sb = lambda S, B: np.stack([S, B], axis=-1).astype(np.uint16).view(np.uint8).reshape(-1)

    def swizzled(codes):
        rows, nb = codes.shape
        ch = codes.reshape(rows, nb // 16, 16)
        res = np.empty_like(ch)
        for i in range(rows):
            for c in range(nb // 16):
                res[i, (c & ~7) | ((c ^ i) & 7)] = ch[i, c]
        return res.reshape(-1)

    rP = m["router"][0].view(np.uint8).reshape(E, H)
    rS, rB = m["router"][1].reshape(E, GH), m["router"][2].reshape(E, GH)
    for r in range(8):
        rows = slice(Rr * r, Rr * r + Rr)
        out += [swizzled(rP[rows]), sb(rS[rows], rB[rows])]

    def mat(name, e, rows_n, cols):
        P, S, B = m[name]
        P = P.reshape(-1, rows_n, cols // 8)[e if P.ndim == 3 else 0]
        S = S.reshape(-1, rows_n, cols // 64)[e if S.ndim == 3 else 0]
        Bb = B.reshape(-1, rows_n, cols // 64)[e if B.ndim == 3 else 0]
        return P.view(np.uint8).reshape(rows_n, cols // 2), S, Bb
    for e in range(E + 1):
        g_, u_, d_ = ("gate", "up", "down") if e < E else ("sh_gate", "sh_up", "sh_down")
        gP, gS, gB = mat(g_, e, I, H)
        uP, uS, uB = mat(u_, e, I, H)
        dP, dS, dB = mat(d_, e, H, I)
        for g in range(GI):
            for r in range(8):
                rows = slice(64 * g + 8 * r, 64 * g + 8 * r + 8)
                out += [swizzled(gP[rows]), sb(gS[rows], gB[rows])]
                out += [swizzled(uP[rows]), sb(uS[rows], uB[rows])]
                dr = slice(Hc * r, Hc * r + Hc)
                out += [dP[dr, 32 * g:32 * g + 32].reshape(-1), sb(dS[dr, g], dB[dr, g])]
    return np.concatenate(out)


def test_pack_layout_bit_exact(cuda_dev):
    E, H, I = 16, 512, 128
    ms, stack = make_stack(91, 1, E, H, I, 4)
    got = stack.packed[0].cpu().numpy()
    want = expected_pack(ms[0], E, H, I)
    assert got.size == want.size
    assert np.array_equal(got, want)


@pytest.mark.slow
def test_fp16_overflow_matches_oracle_rounding(cuda_dev):
    """Layer 3 of the seed-0 decode workload: with the stated value ranges
    (fp16 bias ~U(-0.1, 0.1), so every weight row has a positive mean and a
    common component proportional to the sum of x), 328 of its 2816 outputs
    exceed the fp16 range.  Fused and per-layer paths must round them to
    +-inf exactly where rounding the fp64 oracle to fp16 does, and stay
    within tolerance everywhere else."""
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_TOPK
    m = synth.moe_layer(0, 3)
    G = qmoe.MoELayer.from_numpy(m, E, H, I)
    x16 = synth.activations(0, 1, H, layer=3)
    _, oidx, owt = oracle.router(*m["router"], E, H, 8, x16, k)
    y64, y16 = oracle.Layer(m, E, H, I).moe(x16, oidx, owt)
    want = y16[0].view(np.float16).astype(np.float64)
    assert np.isinf(want).sum() > 0
    y, idx, _, _ = run(qmoe.DecodeStack([G], k), x16, E, k)
    assert np.array_equal(idx[0], oidx[0])
    xd = torch.from_numpy(x16.view(np.float16).copy()).cuda()
    i2 = torch.empty(1, k, dtype=torch.int32, device="cuda")
    w2 = torch.empty(1, k, dtype=torch.float32, device="cuda")
    qmoe.moe_router_topk(G.router, xd, k, i2, w2)
    y2 = f16_bits(qmoe.moe_expert_qmlp(G, xd[0], i2.reshape(-1), w2.reshape(-1)))
    for got, what in ((y[0], "fused"), (y2, "per-layer")):
        g = got.view(np.float16).astype(np.float64)
        assert np.array_equal(np.isinf(g), np.isinf(want)), what
        assert np.array_equal(np.sign(g[np.isinf(g)]), np.sign(want[np.isinf(want)])), what
        fin = np.isfinite(want)
        den = np.maximum(np.abs(y64[0][fin]), 1e-2 * np.abs(y64[0][fin]).max())
        assert (np.abs(g[fin] - y64[0][fin]) / den).max() <= REL_TOL, what


def test_x_alignment_rule(cuda_dev):
    """The fused decode reads x 16 bytes at a time: an x that starts one fp16
    element into its buffer is refused before any launch (QMOE_ERR_ALIGNMENT),
    and the same values 16-byte aligned go through."""
    E, H, I, k, n = 16, 256, 64, 4, 2
    ms, stack = make_stack(5, n, E, H, I, k)
    x16 = np.concatenate([synth.activations(9 + l, 1, H, layer=l) for l in range(n)])
    buf = torch.empty(n * H + 8, dtype=torch.float16, device="cuda")
    buf[1:1 + n * H] = torch.from_numpy(x16.view(np.float16).copy()).cuda().reshape(-1)
    xbad = buf[1:1 + n * H].view(n, H)
    assert xbad.data_ptr() % 16 == 2
    with pytest.raises(qmoe.QmoeError) as e:
        qmoe.moe_decode_layers(stack, xbad)
    assert e.value.code == -2
    y, idx, wt, lg = run(stack, x16, E, k)
    check_layers(ms, E, H, I, k, x16, y, idx, wt, lg)
