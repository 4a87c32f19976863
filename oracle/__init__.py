"""Plain fp64 CPU oracle for the affine-quantized GEMV / MoE-layer path.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA library and never imports it.

The arithmetic lives in ``oracle.c`` (fp64, loops in index order, one rounding
at the end); this module only marshals numpy arrays through ctypes.  Arrays of
fp16 values travel as their uint16 bit patterns so that the oracle, not numpy,
decodes them.

Sources of the definitions (page titles and sections):
  * TurboFieldfare article (jeff.news), "성능과 제약" (performance and
    constraints): MLX affine 4-bit weights, group 64; 8-bit router.
  * same article, "내부 구조가 진짜 흥미로운 부분" (internal structure): top-8
    routed experts, a resident shared expert whose output is added to the
    routed output, prefill in chunks of at most 128 tokens.
"""
import ctypes
import numpy as np

from .build import build as _build

_lib = None
_libs = {}
_threads = False


def use_threads(on=True):
    """Route later oracle calls to the OpenMP build of the same source (its
    output rows split over threads, bit-identical results); only the
    multi-threaded CPU baseline uses it."""
    global _threads, _lib
    _threads = bool(on)
    _lib = None


class OrMat(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p)]


class OrLayer(ctypes.Structure):
    _fields_ = [("gate", OrMat), ("up", OrMat), ("down", OrMat),
                ("sh_gate", OrMat), ("sh_up", OrMat), ("sh_down", OrMat),
                ("E", ctypes.c_int64), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
                ("bits", ctypes.c_int64)]


def lib():
    global _lib
    if _lib is None and _threads in _libs:
        _lib = _libs[_threads]
    if _lib is None:
        L = ctypes.CDLL(_build(threads=_threads))
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.or_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_f16_to_f64.restype = ctypes.c_double
        L.or_f64_to_f16.argtypes = [ctypes.c_double]
        L.or_f64_to_f16.restype = ctypes.c_uint16
        L.or_unpack.argtypes = [p, i64, i64, ctypes.c_int, p]
        L.or_pack.argtypes = [p, i64, i64, ctypes.c_int, p]
        L.or_dequant.argtypes = [p, p, p, i64, i64, ctypes.c_int, p]
        L.or_qgemv.argtypes = [p, p, p, i64, i64, ctypes.c_int, p, i64, p, p]
        L.or_router.argtypes = [p, p, p, i64, i64, ctypes.c_int, p, i64, i64, p, p, p]
        L.or_topk_from_logits.argtypes = [p, i64, i64, i64, p, p]
        L.or_expert.argtypes = [ctypes.POINTER(OrLayer), i64, p, p]
        L.or_moe_layer.argtypes = [ctypes.POINTER(OrLayer), p, i64, p, p, i64, p, p]
        L.or_group.argtypes = [p, i64, i64, i64, p, p, p]
        L.or_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_f64.restype = ctypes.c_double
        L.or_rht32.argtypes = [p, p, i64, i64, p]
        L.or_dequant_fmt.argtypes = [p, p, i64, i64, ctypes.c_int, p]
        L.or_qgemv_fmt.argtypes = [p, p, i64, i64, ctypes.c_int, p, ctypes.c_int, p, i64, p, p]
        L.or_lfu_step.argtypes = [i64, p, p, p, i64, p, p, p]
        L.or_lfu_step.restype = i64
        for name in ("or_unpack", "or_pack", "or_dequant", "or_qgemv", "or_router",
                     "or_topk_from_logits", "or_expert", "or_moe_layer", "or_group"):
            getattr(L, name).restype = ctypes.c_int
        _lib = _libs[_threads] = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (np.dtype(dtype), a.dtype))
    return a


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (rc=%d)" % (what, rc))


# ---------------------------------------------------------------- fp16 ------
def f16_to_f64(bits):
    """fp16 bit patterns (uint16 array) -> fp64 values, decoded by the oracle."""
    bits = np.asarray(bits, dtype=np.uint16)
    f = lib().or_f16_to_f64
    return np.array([f(int(b)) for b in bits.ravel()], dtype=np.float64).reshape(bits.shape)


def f64_to_f16(values):
    """fp64 values -> fp16 bit patterns, round to nearest even."""
    values = np.asarray(values, dtype=np.float64)
    f = lib().or_f64_to_f16
    return np.array([f(float(v)) for v in values.ravel()], dtype=np.uint16).reshape(values.shape)


# ------------------------------------------------------------- packing ------
def unpack(packed, N, K, bits):
    packed = _c(packed, np.uint32)
    out = np.empty((N, K), dtype=np.uint8)
    _check(lib().or_unpack(_ptr(packed), N, K, bits, _ptr(out)), "unpack")
    return out


def pack(codes, bits):
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    out = np.empty((N, K * bits // 32), dtype=np.uint32)
    _check(lib().or_pack(_ptr(codes), N, K, bits, _ptr(out)), "pack")
    return out


def dequant(packed, scales, biases, N, K, bits):
    """Dense fp64 [N][K] matrix w = scale*q + bias."""
    packed, scales, biases = _c(packed, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    out = np.empty((N, K), dtype=np.float64)
    _check(lib().or_dequant(_ptr(packed), _ptr(scales), _ptr(biases), N, K, bits, _ptr(out)),
           "dequant")
    return out


# --------------------------------------------------------------- qGEMV ------
def qgemv(packed, scales, biases, N, K, bits, x16):
    """y = W x for x [B][K] (fp16 bits). Returns (y64 [B][N] fp64, y16 [B][N] fp16 bits)."""
    packed, scales, biases = _c(packed, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    x16 = _c(np.atleast_2d(x16), np.uint16)
    B = x16.shape[0]
    assert x16.shape[1] == K
    y64 = np.empty((B, N), dtype=np.float64)
    y16 = np.empty((B, N), dtype=np.uint16)
    _check(lib().or_qgemv(_ptr(packed), _ptr(scales), _ptr(biases), N, K, bits, _ptr(x16), B,
                          _ptr(y64), _ptr(y16)), "qgemv")
    return y64, y16


# -------------------------------------------------------------- router ------
FMT_ZP4, FMT_SYM8 = 1, 2


def bf16_to_f64(bits):
    """bf16 bit patterns -> fp64 values (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return np.array([lib().or_bf16_to_f64(int(v)) for v in b.ravel()], dtype=np.float64).reshape(
        b.shape)


def rht32(x, signs, K):
    """The block-32 random Hadamard rotation of x [B][K] (fp64 values);
    signs: uint32 [K/32] or None (D = I)."""
    x = _c(np.atleast_2d(x), np.float64)
    B = x.shape[0]
    out = np.empty((B, K), np.float64)
    s = None if signs is None else _c(signs, np.uint32)
    _check(lib().or_rht32(_ptr(x), None if s is None else _ptr(s), B, K, _ptr(out)), "or_rht32")
    return out


def dequant_fmt(packed, params, N, K, fmt):
    W = np.empty((N, K), np.float64)
    _check(lib().or_dequant_fmt(_ptr(_c(packed, np.uint32)), _ptr(_c(params, np.uint32)), N, K,
                                fmt, _ptr(W)), "or_dequant_fmt")
    return W


def qgemv_fmt(packed, params, N, K, fmt, x16, signs=None, rotate=False):
    """Format-variant qGEMV: returns (y64 [B][N], y16 bits [B][N])."""
    x = _c(np.atleast_2d(x16), np.uint16)
    B = x.shape[0]
    y64 = np.empty((B, N), np.float64)
    y16 = np.empty((B, N), np.uint16)
    s = None if signs is None else _c(signs, np.uint32)
    _check(lib().or_qgemv_fmt(_ptr(_c(packed, np.uint32)), _ptr(_c(params, np.uint32)), N, K, fmt,
                              None if s is None else _ptr(s), int(bool(rotate)), _ptr(x), B,
                              _ptr(y64), _ptr(y16)), "or_qgemv_fmt")
    return y64, y16


def router(packed, scales, biases, E, K, bits, x16, top_k):
    """Returns (logits64 [T][E], idx [T][k] int32, wt [T][k] fp64)."""
    packed, scales, biases = _c(packed, np.uint32), _c(scales, np.uint16), _c(biases, np.uint16)
    x16 = _c(np.atleast_2d(x16), np.uint16)
    T = x16.shape[0]
    logits = np.empty((T, E), dtype=np.float64)
    idx = np.empty((T, top_k), dtype=np.int32)
    wt = np.empty((T, top_k), dtype=np.float64)
    _check(lib().or_router(_ptr(packed), _ptr(scales), _ptr(biases), E, K, bits, _ptr(x16), T,
                           top_k, _ptr(logits), _ptr(idx), _ptr(wt)), "router")
    return logits, idx, wt


def topk_from_logits(logits32, top_k):
    """The oracle's selection (softmax, top-k with lowest-index ties, renorm)
    applied to given fp32 logits [T][E]."""
    logits32 = _c(np.atleast_2d(logits32), np.float32)
    T, E = logits32.shape
    idx = np.empty((T, top_k), dtype=np.int32)
    wt = np.empty((T, top_k), dtype=np.float64)
    _check(lib().or_topk_from_logits(_ptr(logits32), T, E, top_k, _ptr(idx), _ptr(wt)), "topk")
    return idx, wt


# ----------------------------------------------------------- MoE layer ------
class Layer:
    """Host copy of one MoE layer in the packed format, as the oracle reads it.

    ``mats`` maps gate/up/down/sh_gate/sh_up/sh_down to (packed, scales,
    biases) numpy arrays; routed matrices are stacked over E experts."""

    def __init__(self, mats, E, H, I, bits=4):
        self.E, self.H, self.I, self.bits = E, H, I, bits
        self._keep = {}
        fields = {}
        for name in ("gate", "up", "down", "sh_gate", "sh_up", "sh_down"):
            P, S, B = mats[name]
            P, S, B = _c(P, np.uint32), _c(S, np.uint16), _c(B, np.uint16)
            self._keep[name] = (P, S, B)
            fields[name] = OrMat(P.ctypes.data, S.ctypes.data, B.ctypes.data)
        self.c = OrLayer(fields["gate"], fields["up"], fields["down"], fields["sh_gate"],
                         fields["sh_up"], fields["sh_down"], E, H, I, bits)

    def expert(self, e, x16):
        """Expert e (e < 0: the shared expert) on one token; fp64 [H]."""
        x16 = _c(np.asarray(x16).reshape(-1), np.uint16)
        r = np.empty(self.H, dtype=np.float64)
        _check(lib().or_expert(ctypes.byref(self.c), e, _ptr(x16), _ptr(r)), "expert")
        return r

    def moe(self, x16, idx, wt):
        """y = shared(x) + sum_j wt_j expert_{idx_j}(x) for x [T][H] fp16 bits.
        Returns (y64 [T][H], y16 [T][H] fp16 bits)."""
        x16 = _c(np.atleast_2d(x16), np.uint16)
        T = x16.shape[0]
        idx = np.ascontiguousarray(np.atleast_2d(idx), dtype=np.int32)
        wt = _c(np.atleast_2d(np.asarray(wt, dtype=np.float64)), np.float64)
        k = idx.shape[1]
        y64 = np.empty((T, self.H), dtype=np.float64)
        y16 = np.empty((T, self.H), dtype=np.uint16)
        _check(lib().or_moe_layer(ctypes.byref(self.c), _ptr(x16), T, _ptr(idx), _ptr(wt), k,
                                  _ptr(y64), _ptr(y16)), "moe_layer")
        return y64, y16


def group(idx, E):
    """Counting sort of (token, slot) pairs by expert.
    Returns (counts [E], offsets [E+1], pairs [T*k]) as int32."""
    idx = _c(np.atleast_2d(idx), np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    pairs = np.empty(T * k, dtype=np.int32)
    _check(lib().or_group(_ptr(idx), T, k, E, _ptr(counts), _ptr(offsets), _ptr(pairs)), "group")
    return counts, offsets, pairs


class LfuCache:
    """The per-layer LFU expert cache plan (see or_lfu_step in oracle.c)."""

    def __init__(self, nslots=16):
        self.nslots = nslots
        self.expert = np.full(nslots, -1, np.int32)
        self.count = np.zeros(nslots, np.int64)

    def step(self, ids):
        """-> (slot_of [k], misses [(expert, slot), ...])."""
        ids = _c(np.asarray(ids, np.int32), np.int32)
        k = ids.size
        slot_of = np.empty(k, np.int32)
        me = np.empty(max(k, 1), np.int32)
        ms = np.empty(max(k, 1), np.int32)
        nm = lib().or_lfu_step(self.nslots, _ptr(self.expert), _ptr(self.count), _ptr(ids), k,
                               _ptr(slot_of), _ptr(me), _ptr(ms))
        if nm < 0:
            raise ValueError("k > nslots, nslots outside 1..256, or repeated ids")
        return slot_of, list(zip(me[:nm].tolist(), ms[:nm].tolist()))

