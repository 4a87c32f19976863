"""Pins of the format-variant oracle (zero-point 4-bit and symmetric 8-bit
with bf16 scales, block-32 random Hadamard rotation of the input) to facts
that do not come from the oracle: numpy's bit-level bf16 decode, SciPy's
Hadamard matrix, hand-built codes with known weights, closed forms and an
independent numpy construction of the whole product.

Each test names the mistake it is there to catch.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from moe_expert_gemv_b200 import synth


def _np_bf16(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _np_rotate(x, signs, K):
    """R x with R = blockdiag(H_32 D / sqrt(32)) from SciPy's Hadamard."""
    H = scipy.linalg.hadamard(32).astype(np.float64) / np.sqrt(32.0)
    x = np.atleast_2d(np.asarray(x, np.float64))
    out = np.empty_like(x)
    for blk in range(K // 32):
        d = np.ones(32)
        if signs is not None:
            d = np.where((int(signs[blk]) >> np.arange(32)) & 1, -1.0, 1.0)
        out[:, blk * 32:(blk + 1) * 32] = (x[:, blk * 32:(blk + 1) * 32] * d) @ H.T
    return out


def _np_weights(P, params, N, K, fmt):
    """Independent numpy decode of a format-variant matrix."""
    bits = 4 if fmt == oracle.FMT_ZP4 else 8
    per = 32 // bits
    shifts = (bits * np.arange(per)).astype(np.uint32)
    q = ((P[:, :, None] >> shifts) & ((1 << bits) - 1)).reshape(N, K).astype(np.int64)
    if fmt == oracle.FMT_SYM8:
        q = np.where(q >= 128, q - 256, q)
    s = np.repeat(_np_bf16(params & 0xFFFF), 64, axis=1)
    z = np.repeat(((params >> 16) & 0xFF).astype(np.int64), 64, axis=1)
    return s * (q - z) if fmt == oracle.FMT_ZP4 else s * q


def test_bf16_decode_exhaustive():
    """catches: a wrong shift or byte order in the bf16 decode."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f64(bits)
    want = _np_bf16(bits)
    both_nan = np.isnan(got) & np.isnan(want)
    assert np.array_equal(got[~both_nan], want[~both_nan])
    assert np.array_equal(np.isnan(got), np.isnan(want))


def test_rotation_matches_scipy_hadamard():
    """catches: a wrong Hadamard sign pattern, a missing 1/sqrt(32), signs
    applied after instead of before the transform, a wrong sign-bit order."""
    g = np.random.default_rng(5)
    K = 128
    x = g.standard_normal((3, K))
    signs = g.integers(0, 2 ** 32, K // 32, dtype=np.uint64).astype(np.uint32)
    for s in (None, signs):
        assert np.allclose(oracle.rht32(x, s, K), _np_rotate(x, s, K), rtol=0, atol=1e-12)


def test_rotation_closed_forms():
    """catches: a non-orthonormal transform; a per-block mix-up."""
    K = 64
    e0 = np.zeros((1, K))
    e0[0, 0] = 1.0
    r = oracle.rht32(e0, None, K)
    assert np.allclose(r[0, :32], 1.0 / np.sqrt(32.0), atol=1e-15)
    assert np.all(r[0, 32:] == 0.0)                      # the second block is untouched
    g = np.random.default_rng(6)
    x = g.standard_normal((4, K))
    signs = g.integers(0, 2 ** 32, K // 32, dtype=np.uint64).astype(np.uint32)
    rx = oracle.rht32(x, signs, K)
    for blk in range(K // 32):                            # norm preserved block by block
        sl = slice(32 * blk, 32 * blk + 32)
        assert np.allclose(np.linalg.norm(rx[:, sl], axis=1), np.linalg.norm(x[:, sl], axis=1),
                           rtol=1e-13)


def test_zero_point_codes_give_zero_weights():
    """catches: w = s*q + z or a dropped zero point."""
    N, K = 4, 128
    z = np.arange(N * (K // 64), dtype=np.uint32).reshape(N, K // 64) % 16
    codes = np.repeat(z, 64, axis=1).astype(np.uint8)
    P = oracle.pack(codes, 4)
    params = synth.to_bf16_bits(np.full((N, K // 64), 0.5)).astype(np.uint32) | (z << 16)
    W = oracle.dequant_fmt(P, params, N, K, oracle.FMT_ZP4)
    assert np.all(W == 0.0)
    # one step above the zero point is exactly the scale
    P1 = oracle.pack(np.minimum(codes + 1, 15).astype(np.uint8), 4)
    W1 = oracle.dequant_fmt(P1, params, N, K, oracle.FMT_ZP4)
    assert np.all(W1[np.repeat(z, 64, axis=1) < 15] == 0.5)


def test_symmetric_8bit_hand_word():
    """catches: unsigned instead of two's-complement codes, byte order."""
    # bytes LSB first: 0x01 -> 1, 0xFF -> -1, 0x80 -> -128, 0x7F -> 127
    P = np.full((1, 16), 0x7F80FF01, np.uint32)
    params = np.full((1, 1), synth.to_bf16_bits(0.25), np.uint32)
    W = oracle.dequant_fmt(P, params, 1, 64, oracle.FMT_SYM8)
    assert np.array_equal(W[0, :4], np.array([1.0, -1.0, -128.0, 127.0]) * 0.25)


@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("rotate", [False, True])
def test_qgemv_fmt_brute_force(fmt, rotate):
    """catches: any mix-up between decode, rotation and product."""
    N, K, B = 24, 192, 3
    P, params, signs = synth.qmatrix_fmt(synth.rng(fmt, int(rotate), 9), N, K, fmt)
    x16 = synth.activations(40 + fmt, B, K)
    y64, y16 = oracle.qgemv_fmt(P, params, N, K, fmt, x16, signs, rotate)
    x = x16.view(np.float16).astype(np.float64)
    xr = _np_rotate(x, signs, K) if rotate else x
    want = xr @ _np_weights(P, params, N, K, fmt).T
    assert np.allclose(y64, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.array_equal(y16, want.astype(np.float16).view(np.uint16)) or \
        np.abs(y16.view(np.float16).astype(np.float64) - want).max() <= \
        np.abs(want).max() * 2 ** -10
