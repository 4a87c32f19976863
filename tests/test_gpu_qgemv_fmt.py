"""qgemv_fmt (zero-point 4-bit / symmetric 8-bit with bf16 scales, optional
block-32 Hadamard rotation of the input) on the GPU against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, assert_close_rows, f16_bits, to_dev_f16

pytestmark = pytest.mark.gpu


def run(P, params, signs, N, K, fmt, rotate, x16):
    W = qmoe.QMatrixFmt.from_numpy(P, params, signs, N, K, fmt, rotate=rotate)
    y = qmoe.qgemv_fmt(W, to_dev_f16(x16))
    assert qmoe.qmoe_check_status() == 0
    return f16_bits(y)


@pytest.mark.parametrize("fmt", [qmoe.FMT_ZP4_BF16, qmoe.FMT_SYM8_BF16])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("N,K", [(512, 1024), (200, 1024), (136, 128), (24, 192), (1000, 4096)])
def test_formats_against_oracle(cuda_dev, fmt, rotate, N, K):
    """Both formats, with and without the rotation; swizzled tensor-copy
    tiles (K*bits/32 % 32 == 0) and padded row copies; row tails."""
    P, params, signs = synth.qmatrix_fmt(synth.rng(N, K, fmt, 3), N, K, fmt)
    for Bt in (1, 3, 8):
        x16 = synth.activations(N + K + Bt + 7 * fmt, Bt, K)
        y = run(P, params, signs, N, K, fmt, rotate, x16)
        y64, _ = oracle.qgemv_fmt(P, params, N, K, fmt, x16, signs, rotate)
        assert_close_rows(y.view(np.float16), y64,
                          what="fmt %d rot %d N=%d K=%d B=%d" % (fmt, rotate, N, K, Bt))


@pytest.mark.parametrize("fmt", [qmoe.FMT_ZP4_BF16, qmoe.FMT_SYM8_BF16])
def test_small_m_batches(cuda_dev, fmt):
    N, K = 200, 1024
    P, params, signs = synth.qmatrix_fmt(synth.rng(N, K, fmt, 12), N, K, fmt)
    for Bt in (13, 32):
        x16 = synth.activations(N + Bt + 5 * fmt, Bt, K)
        y = run(P, params, signs, N, K, fmt, True, x16)
        y64, _ = oracle.qgemv_fmt(P, params, N, K, fmt, x16, signs, True)
        assert_close_rows(y.view(np.float16), y64, what="fmt %d B=%d" % (fmt, Bt))


@pytest.mark.slow
@pytest.mark.parametrize("fmt", [qmoe.FMT_ZP4_BF16, qmoe.FMT_SYM8_BF16])
def test_k4096_shapes_sampled_rows(cuda_dev, fmt):
    """N=14336, K=4096, batch 8 with the rotation: every output of 256
    sampled rows against the oracle (the oracle runs on those rows only)."""
    N, K, Bt = 14336, 4096, 8
    P, params, signs = synth.qmatrix_fmt(synth.rng(N, K, fmt, 4), N, K, fmt)
    x16 = synth.activations(11 + fmt, Bt, K)
    y = run(P, params, signs, N, K, fmt, True, x16).view(np.float16)
    rows = np.random.default_rng(fmt).choice(N, 256, replace=False)
    rows.sort()
    y64, _ = oracle.qgemv_fmt(P[rows], params[rows], len(rows), K, fmt, x16, signs, True)
    assert_close_rows(y[:, rows], y64, what="K=4096 shape fmt %d" % fmt)


def test_zero_input_and_zero_codes(cuda_dev):
    """x = 0 gives +0 everywhere.  Codes at the zero point are zero weights;
    the folded form s*sum(q x) - s*z*sum(x) cancels them up to fp32 rounding
    of the two sums, so y stays below 1e-4 of an ordinary output."""
    N, K = 64, 256
    P, params, signs = synth.qmatrix_fmt(synth.rng(5), N, K, qmoe.FMT_ZP4_BF16)
    y = run(P, params, signs, N, K, qmoe.FMT_ZP4_BF16, True, np.zeros((2, K), np.uint16))
    assert np.all(y == 0)
    x16 = synth.activations(6, 3, K)
    typical = np.abs(run(P, params, signs, N, K, qmoe.FMT_ZP4_BF16, True, x16)
                     .view(np.float16).astype(np.float64)).max()
    z = (params >> 16) & 0xF
    Pz = oracle.pack(np.repeat(z, 64, axis=1).astype(np.uint8), 4)
    y = run(Pz, params, signs, N, K, qmoe.FMT_ZP4_BF16, True, x16)
    assert np.abs(y.view(np.float16).astype(np.float64)).max() <= 1e-4 * typical


def test_bad_format_and_alignment_rejected(cuda_dev):
    N, K = 16, 128
    P, params, signs = synth.qmatrix_fmt(synth.rng(7), N, K, qmoe.FMT_ZP4_BF16)
    W = qmoe.QMatrixFmt.from_numpy(P, params, signs, N, K, qmoe.FMT_ZP4_BF16)
    W.c.format = 9
    with pytest.raises(qmoe.QmoeError):
        qmoe.qgemv_fmt(W, torch.zeros(1, K, dtype=torch.float16, device="cuda"))
    W.c.format = qmoe.FMT_ZP4_BF16
    buf = torch.zeros(K + 1, dtype=torch.float16, device="cuda")
    x = buf[1:].view(1, K)   # 2-byte aligned only: the rotation needs 16-byte aligned x
    with pytest.raises(qmoe.QmoeError):
        qmoe.qgemv_fmt(W, x)


@pytest.mark.parametrize("fmt", [qmoe.FMT_ZP4_BF16, qmoe.FMT_SYM8_BF16])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("N,K,Bt", [(256, 4096, 9), (200, 2048, 16), (1000, 4096, 29),
                                    (512, 8192, 32)])
def test_small_m_one_pass(cuda_dev, fmt, rotate, N, K, Bt):
    """Batch 9..32 of the format variants in one pass over the weights
    (qgemv_fmt_ws; K split into slices whose x, or rotated x hi/lo pair,
    fits on chip): every row against the oracle, and the 8-row-slice path
    on the same inputs agrees within the tolerance."""
    P, params, signs = synth.qmatrix_fmt(synth.rng(N, K, fmt, Bt, 31), N, K, fmt)
    x16 = synth.activations(N + Bt + 7 * fmt, Bt, K)
    W = qmoe.QMatrixFmt.from_numpy(P, params, signs, N, K, fmt, rotate=rotate)
    xd = torch.from_numpy(x16.view(np.float16).copy()).cuda()
    need = qmoe.lib().qgemv_fmt_workspace_bytes(N, K, fmt, int(rotate), Bt)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    y1 = qmoe.qgemv_fmt(W, xd, workspace=ws)
    assert qmoe.qmoe_check_status() == 0
    y0 = qmoe.qgemv_fmt(W, xd, one_pass=False)
    y64, _ = oracle.qgemv_fmt(P, params, N, K, fmt, x16, signs, rotate)
    what = "one-pass fmt %d rot %d N=%d K=%d B=%d" % (fmt, rotate, N, K, Bt)
    assert_close_rows(y1.cpu().numpy(), y64, what=what)
    assert_close_rows(y1.cpu().numpy(), y0.cpu().numpy().astype(np.float64), what=what + " vs slices")
    if need:   # the workspace's counters are back at zero
        assert torch.count_nonzero(ws[:65536]) == 0
