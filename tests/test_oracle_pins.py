"""Pins of the CPU oracle to facts that do not come from the oracle itself:
hand-derived fixtures (tests/golden), closed forms, invariants, special cases
that reduce to a library routine, and brute force on tiny inputs.

Each test names the mistake it is there to catch.
"""
import os

import numpy as np
import pytest

import oracle
from moe_expert_gemv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _np_f16(bits):
    """Independent fp16 decode (numpy's), used to cross-check the oracle's."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _np_dense(P, S, B, N, K, bits):
    """Dense fp64 matrix from the oracle's (pinned) unpack and numpy's fp16
    decode: a second construction of the dequantised weights."""
    q = oracle.unpack(P, N, K, bits).astype(np.float64)
    s = np.repeat(_np_f16(S).reshape(N, K // 64), 64, axis=1)
    b = np.repeat(_np_f16(B).reshape(N, K // 64), 64, axis=1)
    return s * q + b


# ------------------------------------------------------------------ fp16 ----
def test_f16_decode_exhaustive():
    """All 65,536 fp16 patterns decode like numpy's float16 (catches a wrong
    exponent bias, a subnormal slip or a sign error)."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f64(allbits)
    ref = allbits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_f16_encode_round_to_nearest_even():
    """fp64 -> fp16 matches numpy (correctly rounded, ties to even) on every
    finite half, every midpoint between neighbours, and random doubles."""
    finite = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    finite = finite[np.isfinite(finite)].astype(np.float64)
    srt = np.unique(finite)
    mids = (srt[:-1] + srt[1:]) / 2.0
    g = np.random.default_rng(7)
    rnd = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-9, 6, 20000),
                          [65504.0, 65519.999, 65520.0, 1e6, -1e6, 2.0 ** -25, 2.0 ** -26,
                           3 * 2.0 ** -26, 0.0, -0.0]])
    for vals in (finite, mids, rnd):
        ours = oracle.f64_to_f16(vals)
        with np.errstate(over="ignore"):
            ref = vals.astype(np.float16).view(np.uint16)
        assert np.array_equal(ours, ref)


# --------------------------------------------------------------- packing ----
def test_pack_words_golden():
    """Hand-packed words (nibble/byte order, least significant first)."""
    for row in _lines("pack_words.txt"):
        bits, word, codes = int(row[0]), int(row[1], 16), [int(c) for c in row[2:]]
        per = 32 // bits
        assert len(codes) == per
        got = oracle.unpack(np.array([[word]], dtype=np.uint32), 1, per, bits)
        assert got.ravel().tolist() == codes
        back = oracle.pack(np.array([codes], dtype=np.uint8), bits)
        assert int(back[0, 0]) == word


@pytest.mark.parametrize("bits", [4, 8])
def test_pack_unpack_roundtrip(bits):
    g = np.random.default_rng(bits)
    N, K = 13, 192
    codes = g.integers(0, 2 ** bits, (N, K)).astype(np.uint8)
    assert np.array_equal(oracle.unpack(oracle.pack(codes, bits), N, K, bits), codes)
    words = g.integers(0, 2 ** 32, (N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(oracle.pack(oracle.unpack(words, N, K, bits), bits), words)


# --------------------------------------------------------------- dequant ----
def test_dequant_golden():
    """Scale and bias of the right group (catches k/32 vs k/64, scale/bias
    swapped, a dropped bias)."""
    rows = _lines("dequant_example.txt")
    a = [r for r in rows if r[0] == "A"][0]
    s, b, word = float(a[1]), float(a[2]), int(a[3], 16)
    want = [float(v) for v in a[4:]]
    P = np.full((1, 8), word, dtype=np.uint32)
    S = synth.to_f16_bits([[s]])
    Bb = synth.to_f16_bits([[b]])
    W = oracle.dequant(P, S, Bb, 1, 64, 4)
    assert W[0, :8].tolist() == want
    # case B: two groups with different scale/bias
    P = np.concatenate([np.full(8, 0x76543210), np.full(8, 0xFEDCBA98)]).astype(np.uint32)[None]
    S = synth.to_f16_bits([[1.0, 2.0]])
    Bb = synth.to_f16_bits([[0.0, 10.0]])
    W = oracle.dequant(P, S, Bb, 1, 128, 4)
    for r in rows:
        if r[0] == "B":
            assert W[0, int(r[1])] == float(r[2])


# ----------------------------------------------------------------- qGEMV ----
def test_qgemv_closed_form_golden():
    s, b, word, x, y, ybits = _lines("qgemv_closed_form.txt")[0]
    P = np.full((1, 8), int(word, 16), dtype=np.uint32)
    y64, y16 = oracle.qgemv(P, synth.to_f16_bits([[float(s)]]), synth.to_f16_bits([[float(b)]]),
                            1, 64, 4, synth.to_f16_bits(np.full((1, 64), float(x))))
    assert y64[0, 0] == float(y)
    assert int(y16[0, 0]) == int(ybits, 16)


@pytest.mark.parametrize("bits", [4, 8])
def test_qgemv_unit_vectors(bits):
    """x = e_k picks column k: y[n] = fp16(s[n,k/64] q[n,k] + b[n,k/64]) (catches
    a transposed operand or a wrong column/group index)."""
    N, K = 24, 192
    P, S, B = synth.qmatrix(synth.rng(3, bits), N, K, bits)
    W = _np_dense(P, S, B, N, K, bits)
    for k in (0, 1, 7, 8, 63, 64, 100, 191):
        x = np.zeros((1, K))
        x[0, k] = 1.0
        y64, y16 = oracle.qgemv(P, S, B, N, K, bits, synth.to_f16_bits(x))
        assert np.array_equal(y64[0], W[:, k])
        assert np.array_equal(y16[0], W[:, k].astype(np.float16).view(np.uint16))


def test_qgemv_zero_codes_is_bias_only():
    """q = 0 everywhere -> y[n] = sum_g b[n,g] * (sum of x over group g)."""
    N, K = 16, 256
    _, S, B = synth.qmatrix(synth.rng(4), N, K)
    P = np.zeros((N, K // 8), dtype=np.uint32)
    x16 = synth.activations(5, 3, K)
    xs = _np_f16(x16).reshape(3, K // 64, 64).sum(axis=2)           # [B][G]
    want = xs @ _np_f16(B).reshape(N, K // 64).T                      # [B][N]
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    np.testing.assert_allclose(y64, want, rtol=1e-12, atol=1e-12)


def test_qgemv_zero_input_gives_positive_zero():
    N, K = 16, 128
    P, S, B = synth.qmatrix(synth.rng(6), N, K)
    _, y16 = oracle.qgemv(P, S, B, N, K, 4, np.zeros((2, K), dtype=np.uint16))
    assert np.all(y16 == 0)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [64, 128, 192])
def test_qgemv_bruteforce_dense(bits, K):
    """fp64 numpy matmul of the dequantised matrix (library routine) on tiny
    shapes, every batch size 1..8."""
    for N in (1, 5, 17):
        P, S, B = synth.qmatrix(synth.rng(K, N, bits), N, K, bits)
        W = _np_dense(P, S, B, N, K, bits)
        assert np.array_equal(oracle.dequant(P, S, B, N, K, bits), W)
        for Bt in (1, 2, 3, 8):
            x16 = synth.activations(K + N + Bt, Bt, K)
            y64, y16 = oracle.qgemv(P, S, B, N, K, bits, x16)
            ref = _np_f16(x16) @ W.T
            np.testing.assert_allclose(y64, ref, rtol=1e-12, atol=1e-12)
            assert np.array_equal(y16, oracle.f64_to_f16(y64))


# ---------------------------------------------------------------- router ----
def test_topk_ties_golden():
    for row in _lines("topk_ties.txt"):
        bar1 = row.index("|")
        bar2 = row.index("|", bar1 + 1)
        k = int(row[0])
        logits = np.array([[float(v) for v in row[bar1 + 1:bar2]]], dtype=np.float32)
        want = [int(v) for v in row[bar2 + 1:]]
        idx, wt = oracle.topk_from_logits(logits, k)
        assert idx[0].tolist() == want
        assert abs(wt.sum() - 1.0) < 1e-15


def test_router_zero_input_uniform():
    """x = 0 -> every logit 0 -> uniform softmax -> idx 0..7 (lowest index wins
    the 128-way tie) and each weight exactly 1/8."""
    E, K = 128, 2816
    P, S, B = synth.router(1, E, K)
    logits, idx, wt = oracle.router(P, S, B, E, K, 8, np.zeros((1, K), np.uint16), 8)
    assert np.all(logits == 0.0)
    assert idx[0].tolist() == list(range(8))
    assert np.all(wt == 0.125)


def test_router_bruteforce_and_invariants():
    """Small E: the oracle's softmax -> top-k -> renormalise equals a full
    stable sort of the logits and a softmax over the selected logits only
    (closed form of the renormalisation); weights sum to 1, descend."""
    E, K, k = 16, 128, 4
    P, S, B = synth.router(2, E, K)
    x16 = synth.activations(3, 6, K)
    logits, idx, wt = oracle.router(P, S, B, E, K, 8, x16, k)
    W = _np_dense(P, S, B, E, K, 8)
    np.testing.assert_allclose(logits, _np_f16(x16) @ W.T, rtol=1e-12, atol=1e-9)
    for t in range(6):
        order = np.argsort(-logits[t], kind="stable")[:k]
        assert idx[t].tolist() == order.tolist()
        sel = logits[t, order]
        closed = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        np.testing.assert_allclose(wt[t], closed, rtol=1e-12)
        assert abs(wt[t].sum() - 1.0) < 1e-12
        assert np.all(np.diff(wt[t]) <= 0)


def test_router_forced_expert_wins():
    """A router row with a huge bias and an all-positive input takes slot 0
    with weight ~1."""
    E, K = 128, 2816
    P, S, B = synth.router(4, E, K)
    B = B.copy()
    B[77, :] = synth.to_f16_bits(np.full(K // 64, 30.0))
    x16 = synth.to_f16_bits(np.full((1, K), 0.5))
    _, idx, wt = oracle.router(P, S, B, E, K, 8, x16, 8)
    assert idx[0, 0] == 77 and wt[0, 0] > 1 - 1e-9


# -------------------------------------------------------- expert / layer ----
def _tiny_layer(seed, E=4, H=128, I=64):
    m = synth.moe_layer(seed, 0, E=E, H=H, I=I, with_router=False)
    return m, oracle.Layer(m, E, H, I)


def test_layer_bruteforce_dense():
    """E=4, H=128, I=64: numpy matmuls of the dequantised matrices, SwiGLU with
    numpy's exp, weighted sum plus shared -- against the oracle's layer."""
    E, H, I = 4, 128, 64
    m, L = _tiny_layer(11, E, H, I)
    dense = {}
    for name in ("gate", "up", "down"):
        P, S, B = m[name]
        rows, cols = (I, H) if name != "down" else (H, I)
        dense[name] = [_np_dense(P[e], S[e], B[e], rows, cols, 4) for e in range(E)]
    for name in ("sh_gate", "sh_up", "sh_down"):
        P, S, B = m[name]
        rows, cols = (I, H) if name != "sh_down" else (H, I)
        dense[name] = _np_dense(P, S, B, rows, cols, 4)

    def mlp(wg, wu, wd, x):
        g, u = wg @ x, wu @ x
        return wd @ (g / (1.0 + np.exp(-g)) * u)

    x16 = synth.activations(12, 3, H)
    idx = np.array([[2, 0], [3, 1], [1, 2]], dtype=np.int32)
    wt = np.array([[0.7, 0.3], [0.55, 0.45], [0.9, 0.1]])
    y64, y16 = L.moe(x16, idx, wt)
    for t in range(3):
        x = _np_f16(x16[t])
        ref = mlp(dense["sh_gate"], dense["sh_up"], dense["sh_down"], x)
        for j in range(2):
            e = idx[t, j]
            ref = ref + wt[t, j] * mlp(dense["gate"][e], dense["up"][e], dense["down"][e], x)
        np.testing.assert_allclose(y64[t], ref, rtol=1e-11, atol=1e-11)
    assert np.array_equal(y16, oracle.f64_to_f16(y64))


def test_swiglu_closed_form():
    """H = I = 64 with hand-built matrices: gate row i = 2 e_0, up row i = e_0,
    down = identity.  For x = 1.5 e_0: g = 3, u = 1.5, r_n = silu(3) * 1.5 =
    4.5 / (1 + e^-3).  Swapping gate and up would give 3 * silu(1.5)."""
    H = I = 64
    zeros = np.zeros((I, H // 8), np.uint32)
    gate_P = zeros.copy()
    gate_P[:, 0] = 2            # code 2 at k = 0
    up_P = zeros.copy()
    up_P[:, 0] = 1              # code 1 at k = 0
    down_codes = np.eye(H, I, dtype=np.uint8)
    down_P = oracle.pack(down_codes, 4)
    one = synth.to_f16_bits(np.ones((I, 1)))
    zero = synth.to_f16_bits(np.zeros((I, 1)))
    mats = {"gate": (gate_P[None], one[None], zero[None]), "up": (up_P[None], one[None], zero[None]),
            "down": (down_P[None], one[None], zero[None]),
            "sh_gate": (zeros, one, zero), "sh_up": (zeros, one, zero),
            "sh_down": (np.zeros((H, I // 8), np.uint32), one, zero)}
    L = oracle.Layer(mats, 1, H, I)
    x = np.zeros((1, H))
    x[0, 0] = 1.5
    y64, _ = L.moe(synth.to_f16_bits(x), np.array([[0]]), np.array([[1.0]]))
    want = 4.5 / (1.0 + np.exp(-3.0))
    np.testing.assert_allclose(y64[0], np.full(H, want), rtol=1e-15)
    assert abs(want - 3.0 * 1.5 / (1 + np.exp(-1.5))) > 0.1


def test_layer_zero_input_zero_output():
    m, L = _tiny_layer(13)
    y64, y16 = L.moe(np.zeros((1, 128), np.uint16), np.array([[0, 1]]), np.array([[0.5, 0.5]]))
    assert np.all(y64 == 0.0) and np.all(y16 == 0)


def test_layer_one_hot_weight_and_composition():
    """wt = (1, 0) -> y = shared(x) + expert_{idx0}(x)."""
    m, L = _tiny_layer(14)
    x16 = synth.activations(15, 1, 128)
    y64, _ = L.moe(x16, np.array([[3, 1]]), np.array([[1.0, 0.0]]))
    np.testing.assert_allclose(y64[0], L.expert(-1, x16) + L.expert(3, x16), rtol=1e-13)


def test_layer_expert_permutation_invariance():
    """Permuting the stored experts and relabelling idx leaves y unchanged."""
    E, H, I = 4, 128, 64
    m, L = _tiny_layer(16, E, H, I)
    perm = np.array([2, 0, 3, 1])              # new slot p holds old expert perm[p]
    inv = np.argsort(perm)
    m2 = dict(m)
    for name in ("gate", "up", "down"):
        m2[name] = tuple(a[perm] for a in m[name])
    L2 = oracle.Layer(m2, E, H, I)
    x16 = synth.activations(17, 2, H)
    idx = np.array([[1, 3], [0, 2]], dtype=np.int32)
    wt = np.array([[0.6, 0.4], [0.8, 0.2]])
    y_a, _ = L.moe(x16, idx, wt)
    y_b, _ = L2.moe(x16, inv[idx].astype(np.int32), wt)
    np.testing.assert_allclose(y_a, y_b, rtol=1e-14)


# -------------------------------------------------------------- grouping ----
def test_grouping_golden():
    rows = {r[0]: [int(v) for v in r[1:]] for r in _lines("grouping_small.txt")}
    idx = np.array(rows["idx"], dtype=np.int32).reshape(4, 2)
    counts, offsets, pairs = oracle.group(idx, 5)
    assert counts.tolist() == rows["counts"]
    assert offsets.tolist() == rows["offsets"]
    assert pairs.tolist() == rows["pairs"]


def test_grouping_bruteforce_zipf():
    idx, _ = synth.zipf_routing(3)
    counts, offsets, pairs = oracle.group(idx, 128)
    flat = idx.ravel().tolist()
    for e in range(128):
        lst = [i for i in range(len(flat)) if flat[i] == e]
        assert counts[e] == len(lst)
        assert pairs[offsets[e]:offsets[e + 1]].tolist() == lst
    assert sorted(pairs.tolist()) == list(range(idx.size))


def test_zipf_routing_shape():
    """The generator's assignments: distinct experts per token, weights sum to
    one and descend, and the Zipf skew leaves most experts light."""
    idx, wt = synth.zipf_routing(0)
    assert idx.shape == (128, 8) and wt.shape == (128, 8)
    assert all(len(set(r)) == 8 for r in idx.tolist())
    np.testing.assert_allclose(wt.sum(axis=1), 1.0, rtol=1e-6)
    assert np.all(np.diff(wt, axis=1) <= 0)
    c = np.bincount(idx.ravel(), minlength=128)
    assert c.max() > 64 and (c <= 8).sum() > 64


def test_threaded_build_is_bit_identical():
    """The OpenMP build of the oracle (output rows split over threads, used
    only for the multi-threaded CPU baseline) computes every output bit for
    bit like the plain build: each row's sum keeps the index order."""
    from moe_expert_gemv_b200 import synth
    E, H, I = 16, 256, 128
    m = synth.moe_layer(3, 0, E=E, H=H, I=I)
    x16 = synth.activations(3, 5, H)
    P, S, B = synth.dense(3, 96, 512)
    xd = synth.activations(4, 3, 512)
    L = oracle.Layer(m, E, H, I)
    outs = []
    try:
        for threads in (False, True):
            oracle.use_threads(threads)
            lg, idx, wt = oracle.router(*m["router"], E, H, 8, x16, 4)
            y, _ = L.moe(x16, idx, wt)
            q, _ = oracle.qgemv(P, S, B, 96, 512, 4, xd)
            outs.append((lg, idx, wt, y, q))
    finally:
        oracle.use_threads(False)
    for a, b in zip(*outs):
        assert np.array_equal(a, b)
