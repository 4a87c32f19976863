"""The seeded input recipe the parity tests and the benchmark share: the
stated value ranges and distributions, and the facts the design notes quote
about the benchmark's inputs."""
import numpy as np
import pytest

from moe_expert_gemv_b200 import synth


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def nibbles(P):
    w = np.asarray(P, np.uint32).reshape(-1)
    return np.stack([(w >> (4 * i)) & 15 for i in range(8)], axis=1).reshape(-1)


def test_dense_matrix_ranges_and_uniform_codes():
    P, S, B = synth.dense(1, 512, 4096)
    assert P.shape == (512, 512) and S.shape == (512, 64) and B.shape == (512, 64)
    s, b = f16(S), f16(B)
    # fp16 rounding of U(0.005, 0.02) and U(-0.1, 0.1) stays inside the rounded bounds
    assert s.min() >= float(np.float16(0.005)) and s.max() <= float(np.float16(0.02))
    assert b.min() >= float(np.float16(-0.1)) and b.max() <= float(np.float16(0.1))
    assert abs(s.mean() - 0.0125) < 2e-4 and abs(b.mean()) < 3e-3
    q = np.bincount(nibbles(P), minlength=16) / (512 * 4096)
    assert np.all(np.abs(q - 1 / 16) < 2e-3)


def test_router_ranges():
    P, S, B = synth.router(2)
    assert P.shape == (128, 2816 // 4)
    q = np.asarray(P, np.uint32).view(np.uint8)
    assert abs(q.mean() - 127.5) < 1.0
    s, b = f16(S), f16(B)
    assert s.min() >= float(np.float16(0.001)) and s.max() <= float(np.float16(0.004))
    assert b.min() >= float(np.float16(-0.2)) and b.max() <= float(np.float16(0.2))


def test_activations_standard_normal_in_fp16():
    x = f16(synth.activations(0, 64, 4096))
    assert x.shape == (64, 4096)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # exactly the fp16 rounding of the fp64 draw of the same stream
    g = synth.rng(0, 0, 1).standard_normal((64, 4096))
    assert np.array_equal(x, g.astype(np.float16).astype(np.float64))


def test_seeding_is_per_tensor_and_layer():
    a = synth.moe_layer(0, 0, E=4, H=256, I=64)
    b = synth.moe_layer(0, 0, E=4, H=256, I=64)
    c = synth.moe_layer(0, 1, E=4, H=256, I=64)
    for name in a:
        for u, v, w in zip(a[name], b[name], c[name]):
            assert np.array_equal(u, v)
            assert not np.array_equal(u, w)
    assert not np.array_equal(a["gate"][0], a["up"][0])


def test_format_matrices():
    for fmt, bits, lo, hi in ((synth.FMT_ZP4, 4, 0.005, 0.02), (synth.FMT_SYM8, 8, 0.001, 0.004)):
        P, prm, signs = synth.qmatrix_fmt(synth.rng(5, fmt), 64, 1024, fmt)
        assert P.shape == (64, 1024 * bits // 32) and prm.shape == (64, 16) and signs.shape == (32,)
        s = (np.asarray(prm, np.uint32) & 0xFFFF).astype(np.uint32) << 16
        s = s.view(np.float32).astype(np.float64)
        assert s.min() >= lo * (1 - 2 ** -8) and s.max() <= hi * (1 + 2 ** -8)
        z = (np.asarray(prm, np.uint32) >> 16) & 0xFF
        if fmt == synth.FMT_ZP4:
            assert z.max() <= 15 and len(np.unique(z)) == 16
        else:
            assert not z.any()


@pytest.mark.parametrize("rho", [0.0, 0.9, 0.99])
def test_correlated_tokens(rho):
    x = f16(synth.correlated_tokens(0, 400, 2816, rho))
    assert abs(x.std() - 1.0) < 0.02
    c = np.mean([np.corrcoef(x[t], x[t + 1])[0, 1] for t in range(399)])
    assert abs(c - rho) < 0.02


def test_benchmark_chunk_routing_facts():
    """The seed-0 chunk the prefill benchmark times: 122 of 128 experts get
    tokens, 96 of those 1-8 (the light, weight-streaming experts), the
    busiest 109 of the 128 tokens."""
    idx, _ = synth.zipf_routing(0)
    c = np.bincount(idx.ravel(), minlength=128)
    assert (c > 0).sum() == 122
    assert ((c > 0) & (c <= 8)).sum() == 96
    assert c.max() == 109
