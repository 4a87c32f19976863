"""qgemv_affine and the pack helpers on the GPU against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemv_b200 import qmoe, synth
from tests._util import assert_close, assert_close_rows, f16_bits, to_dev_f16

pytestmark = pytest.mark.gpu


def run_qgemv(P, S, B, N, K, bits, x16):
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, bits)
    y = qmoe.qgemv_affine(W, to_dev_f16(x16))
    assert qmoe.qmoe_check_status() == 0
    return f16_bits(y)


@pytest.mark.parametrize("bits", [4, 8])
def test_pack_unpack_bit_exact(cuda_dev, bits):
    g = np.random.default_rng(bits)
    for rows, cols in ((1, 8), (7, 64), (33, 2816)):
        if cols % (32 // bits):
            continue
        codes = g.integers(0, 2 ** bits, (rows, cols)).astype(np.uint8)
        packed = qmoe.qmoe_pack_codes(torch.from_numpy(codes).cuda(), bits)
        want = oracle.pack(codes, bits)
        assert np.array_equal(packed.cpu().numpy().view(np.uint32), want)
        back = qmoe.qmoe_unpack_codes(packed, rows, cols, bits)
        assert np.array_equal(back.cpu().numpy(), codes)
        words = g.integers(0, 2 ** 32, (rows, cols * bits // 32), dtype=np.uint64).astype(np.uint32)
        un = qmoe.qmoe_unpack_codes(torch.from_numpy(words.view(np.int32)).cuda(), rows, cols, bits)
        assert np.array_equal(un.cpu().numpy(), oracle.unpack(words, rows, cols, bits))


def test_small_dense_single_qgemv(cuda_dev):
    """N=512, K=1024, batch 1 (the small dense case)."""
    N, K = 512, 1024
    P, S, B = synth.dense(0, N, K)
    x16 = synth.activations(0, 1, K)
    y = run_qgemv(P, S, B, N, K, 4, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    assert_close(y.view(np.float16), y64, what="N=512 K=1024")


@pytest.mark.slow
@pytest.mark.parametrize("N", [14336, 4096])
@pytest.mark.parametrize("Bt", [1, 4, 8])
def test_k4096_decode_sweep(cuda_dev, N, Bt):
    """K=4096, N in {14336, 4096}, batch 1/4/8, full output against the oracle."""
    K = 4096
    P, S, B = synth.dense(1, N, K)
    x16 = synth.activations(1 + Bt, Bt, K)
    y = run_qgemv(P, S, B, N, K, 4, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    assert_close_rows(y.view(np.float16), y64, what="K=4096 N=%d B=%d" % (N, Bt))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(8, 64), (24, 192), (40, 704), (136, 128), (16, 2816)])
def test_small_and_ragged_shapes(cuda_dev, bits, N, K):
    """Tile tails (N % 16 == 8), a single group, K = 704 (11 groups), every batch."""
    P, S, B = synth.qmatrix(synth.rng(N, K, bits), N, K, bits)
    for Bt in range(1, 9):
        x16 = synth.activations(N + K + Bt, Bt, K)
        y = run_qgemv(P, S, B, N, K, bits, x16)
        y64, _ = oracle.qgemv(P, S, B, N, K, bits, x16)
        assert_close(y.view(np.float16), y64, what="N=%d K=%d B=%d bits=%d" % (N, K, Bt, bits))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(200, 1024), (1000, 4096), (8, 256), (24, 512)])
def test_tensor_copy_tiles_with_row_tail(cuda_dev, bits, N, K):
    """Rows of 128-byte multiples (K % 256 == 0 at 4 bits, K % 128 == 0 at 8
    bits) take whole 16-row tiles in one swizzled tensor copy; the last tile
    here is partial (N % 16 != 0), its missing rows arrive zero-filled."""
    P, S, B = synth.qmatrix(synth.rng(N, K, bits, 7), N, K, bits)
    for Bt in (1, 3, 8):
        x16 = synth.activations(N + K + 10 * Bt, Bt, K)
        y = run_qgemv(P, S, B, N, K, bits, x16)
        y64, _ = oracle.qgemv(P, S, B, N, K, bits, x16)
        assert_close(y.view(np.float16), y64, what="N=%d K=%d B=%d bits=%d" % (N, K, Bt, bits))


@pytest.mark.parametrize("one_pass", [True, False])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(512, 1024), (1000, 4096), (136, 192), (256, 8192)])
def test_small_m_batches(cuda_dev, bits, N, K, one_pass):
    """Batches of 9-32 rows (e.g. the draft tokens a speculative-decoding step
    verifies): the one-pass product (K split into 1, 2, 4 or 8 slices by batch
    and K, ragged last tiles at N=1000; K=192 is a shape it does not take and
    runs the slices) and one launch per 8 rows (ragged last slices)."""
    if not one_pass and bits == 8 and K == 8192:
        pytest.skip("x of 8 rows and a 16-row tile of 8192-wide 8-bit rows exceed shared memory")
    P, S, B = synth.qmatrix(synth.rng(N, K, bits, 11), N, K, bits)
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, bits)
    for Bt in (9, 16, 29, 32):
        x16 = synth.activations(N + 3 * Bt, Bt, K)
        y = f16_bits(qmoe.qgemv_affine(W, to_dev_f16(x16), one_pass=one_pass))
        assert qmoe.qmoe_check_status() == 0
        y64, _ = oracle.qgemv(P, S, B, N, K, bits, x16)
        assert_close_rows(y.view(np.float16), y64,
                          what="N=%d K=%d B=%d bits=%d one_pass=%s" % (N, K, Bt, bits, one_pass))


def test_small_m_workspace_plan(cuda_dev):
    """Workspace sizes of the one-pass product: none for batch <= 8, for one
    slice or for a shape it does not take; partial tiles + counters otherwise."""
    ws = qmoe.lib().qgemv_affine_workspace_bytes
    assert ws(14336, 4096, 4, 8) == 0
    assert ws(512, 1024, 4, 32) == 0          # x of 32 x 1024 fits: one slice
    assert ws(136, 192, 4, 32) == 0           # rows of 96 bytes: not taken
    # K=4096, batch 32: 4 slices of 1024, 64-row tiles, 4 n-tiles
    tiles = 14336 // 64
    assert ws(14336, 4096, 4, 32) == 65536 + tiles * 4 * (4 * 4 * 32) * 16
    assert ws(14336, 4096, 4, 16) > 0


def test_small_m_workspace_shared_across_shapes(cuda_dev):
    """One workspace serving calls of different shapes in turn (the binding
    keeps one per stream): counters live in a fixed region that every call
    leaves at zero, so a shape never reads another's partial tiles as
    counters."""
    cases = [(1000, 4096, 4, 32), (1000, 4096, 8, 9), (256, 8192, 4, 29), (1000, 4096, 8, 32),
             (1000, 4096, 4, 16), (256, 8192, 8, 16)]
    mats = {}
    for rnd in range(2):
        for N, K, bits, Bt in cases:
            if (N, K, bits) not in mats:
                P, S, B = synth.qmatrix(synth.rng(N, K, bits, 21), N, K, bits)
                mats[(N, K, bits)] = (P, S, B, qmoe.QMatrix.from_numpy(P, S, B, N, K, bits))
            P, S, B, W = mats[(N, K, bits)]
            x16 = synth.activations(N + Bt + rnd, Bt, K)
            y = f16_bits(qmoe.qgemv_affine(W, to_dev_f16(x16)))
            y64, _ = oracle.qgemv(P, S, B, N, K, bits, x16)
            assert_close_rows(y.view(np.float16), y64, what="%s round %d" % ((N, K, bits, Bt), rnd))
    assert qmoe.qmoe_check_status() == 0


@pytest.mark.parametrize("Bt", [4, 16, 32])
def test_x_only_2_byte_aligned(cuda_dev, Bt):
    """x may start at any fp16 element: a view one element into its buffer
    (the one-pass product, which loads x 16 bytes at a time, takes the slice
    path for it; the slices stage such an x element by element)."""
    N, K = 1000, 4096
    P, S, B = synth.dense(7, N, K)
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, 4)
    x16 = synth.activations(70 + Bt, Bt, K)
    buf = torch.empty(Bt * K + 1, dtype=torch.float16, device="cuda")
    buf[1:] = to_dev_f16(x16).reshape(-1)
    x = buf[1:].view(Bt, K)
    assert x.data_ptr() % 16 == 2
    y = f16_bits(qmoe.qgemv_affine(W, x))
    assert qmoe.qmoe_check_status() == 0
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    assert_close_rows(y.view(np.float16), y64, what="x at +2 bytes, B=%d" % Bt)


def test_small_m_repeat_bitwise_identical(cuda_dev):
    """The partial tiles are added in slice order whichever CTA finishes last:
    repeated calls give the same bits (and leave the counters at zero)."""
    N, K = 14336, 4096
    P, S, B = synth.dense(1, N, K)
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, 4)
    x = to_dev_f16(synth.activations(5, 32, K))
    y0 = f16_bits(qmoe.qgemv_affine(W, x))
    for _ in range(5):
        assert np.array_equal(f16_bits(qmoe.qgemv_affine(W, x)), y0)
    assert qmoe.qmoe_check_status() == 0


@pytest.mark.slow
@pytest.mark.parametrize("Bt", [16, 32])
def test_k4096_small_m_full(cuda_dev, Bt):
    """K=4096, N=14336 (the decode sweep's large matrix) at batch 16 and 32,
    every output against the oracle, row by row."""
    N, K = 14336, 4096
    P, S, B = synth.dense(1, N, K)
    x16 = synth.activations(40 + Bt, Bt, K)
    y = run_qgemv(P, S, B, N, K, 4, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    assert_close_rows(y.view(np.float16), y64, what="K=4096 N=%d B=%d" % (N, Bt))


def test_zero_input_positive_zero(cuda_dev):
    N, K = 64, 256
    P, S, B = synth.dense(3, N, K)
    y = run_qgemv(P, S, B, N, K, 4, np.zeros((3, K), np.uint16))
    assert np.all(y == 0)


def test_zero_codes_bias_only(cuda_dev):
    N, K = 48, 512
    _, S, B = synth.dense(4, N, K)
    P = np.zeros((N, K // 8), np.uint32)
    x16 = synth.activations(4, 2, K)
    y = run_qgemv(P, S, B, N, K, 4, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, 4, x16)
    assert_close(y.view(np.float16), y64, what="bias only")


@pytest.mark.parametrize("bits", [4, 8])
def test_unit_vectors_exact(cuda_dev, bits):
    """x = e_k: every output is one dequantised weight, exact after fp16 rounding."""
    N, K = 32, 256
    P, S, B = synth.qmatrix(synth.rng(9, bits), N, K, bits)
    ks = [0, 1, 5, 63, 64, 130, 255]
    x = np.zeros((len(ks), K))
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    x16 = synth.to_f16_bits(x)
    y = run_qgemv(P, S, B, N, K, bits, x16)
    _, y16 = oracle.qgemv(P, S, B, N, K, bits, x16)
    assert np.array_equal(y, y16)


def test_repeat_calls_bitwise_identical(cuda_dev):
    N, K = 4096, 4096
    P, S, B = synth.dense(5, N, K)
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, 4)
    x = to_dev_f16(synth.activations(5, 4, K))
    a = qmoe.qgemv_affine(W, x).clone()
    for _ in range(3):
        assert torch.equal(qmoe.qgemv_affine(W, x), a)


@pytest.mark.parametrize("Bt", [6, 8])
def test_long_8bit_rows_take_fewer_rows_per_launch(cuda_dev, Bt):
    """8-bit rows of 8192 columns: 8 rows of x beside a 16-row tile overflow
    shared memory, so each launch takes 4 rows; every output against the
    oracle."""
    N, K = 136, 8192
    P, S, B = synth.qmatrix(synth.rng(N, K, 8, 41), N, K, 8)
    x16 = synth.activations(K + Bt, Bt, K)
    y = run_qgemv(P, S, B, N, K, 8, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, 8, x16)
    assert_close_rows(y.view(np.float16), y64, what="8-bit K=8192 B=%d" % Bt)


def test_rows_too_long_for_one_tile_unsupported(cuda_dev):
    """A 16-row tile of 8-bit rows of 11008 columns plus one row of x does
    not fit in shared memory: UNSUPPORTED, and nothing is launched."""
    N, K = 16, 11008
    P, S, B = synth.qmatrix(synth.rng(N, K, 8, 42), N, K, 8)
    W = qmoe.QMatrix.from_numpy(P, S, B, N, K, 8)
    x = to_dev_f16(synth.activations(43, 1, K))
    with pytest.raises(qmoe.QmoeError) as e:
        qmoe.qgemv_affine(W, x)
    assert e.value.code == qmoe.ERR_UNSUPPORTED
    assert qmoe.qmoe_check_status() == 0


@pytest.mark.parametrize("bits,K", [(8, 10944), (4, 18624)])
def test_longest_rows_one_tile_takes(cuda_dev, bits, K):
    """The longest rows the header documents for one row of x (10944 columns
    at 8 bits, 18624 at 4 bits) run, with a ragged 24-row matrix, against the
    oracle."""
    N = 24
    P, S, B = synth.qmatrix(synth.rng(N, K, bits, 44), N, K, bits)
    x16 = synth.activations(45, 1, K)
    y = run_qgemv(P, S, B, N, K, bits, x16)
    y64, _ = oracle.qgemv(P, S, B, N, K, bits, x16)
    assert_close_rows(y.view(np.float16), y64, what="%d-bit K=%d" % (bits, K))
