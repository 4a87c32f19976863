"""Thin ctypes binding of libqmoe.so (C ABI in include/qmoe.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  Tensors are torch CUDA tensors (PyTorch supplies
device memory and the current stream); fp16 data travels as torch.float16,
packed words as torch.int32 (same bits as the uint32 words of the format).
A non-zero status raises QmoeError.  There is no CPU fallback: if the library
is missing or the device is not an sm_100 GPU the calls fail loudly.
"""
import ctypes
import os

import numpy as np
import torch

from . import build as _build

_lib = None

OK = 0
ERR_INVALID_ARG = -1
ERR_ALIGNMENT = -2
ERR_UNSUPPORTED = -3
ERR_CUDA = -4
ERR_DEVICE_STATUS = -5
ERR_TIMEOUT = -6
ERR_WORKSPACE = -7
DEV_BAD_EXPERT = 0x1
DEV_TIMEOUT = 0x2


class QmoeError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__("%s: %s" % (what, status_string(code)))


class CQMatrix(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("group", ctypes.c_int32)]


class CMoeLayer(ctypes.Structure):
    _fields_ = [("gate", CQMatrix), ("up", CQMatrix), ("down", CQMatrix),
                ("sh_gate", CQMatrix), ("sh_up", CQMatrix), ("sh_down", CQMatrix),
                ("num_experts", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("inter", ctypes.c_int32)]


def lib():
    """Load libqmoe.so (building it first if it has never been built)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not os.path.exists(path):
            _build.build()
        L = ctypes.CDLL(path)
        p, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        sig = {
            "qgemv_affine": [p, p, i32, p, p, p],
            "qgemv_affine_workspace_bytes": [i32, i32, i32, i32],
            "qgemv_affine_ws": [p, p, i32, p, p, sz, p, p],
            "moe_expert_qmlp_ep": [p, p, p, p, i32, i32, i32, p, p, sz, p, p],
            "qmoe_f32_to_f16": [p, p, ctypes.c_int64, p],
            "qgemv_fmt": [p, p, i32, p, p, p],
            "qgemv_fmt_workspace_bytes": [i32, i32, i32, i32, i32],
            "qgemv_fmt_ws": [p, p, i32, p, p, sz, p, p],
            "moe_router_topk": [p, p, i32, i32, p, p, p, p, p],
            "moe_expert_workspace_bytes": [p, i32],
            "moe_expert_qmlp": [p, p, p, p, i32, p, p, sz, p, p],
            "moe_expert_gateup": [p, p, p, i32, p, sz, p, p],
            "moe_expert_down": [p, p, p, i32, p, p, sz, p, p],
            "moe_group_tokens": [p, i32, i32, i32, p, p, p, p, p],
            "moe_decode_pack_bytes": [p],
            "moe_decode_pack_layer": [p, p, p, sz, p],
            "moe_decode_workspace_bytes": [i32, i32, i32, i32],
            "moe_decode_layers": [p, i32, i32, i32, i32, p, i32, p, p, p, p, p, sz, p, p],
            "moe_decode_layers_host": [p, i32, i32, i32, i32, p, p, i32, p, p, p, sz, p, p],
            "moe_prefill_workspace_bytes": [p, i32, i32],
            "moe_prefill_qgemm": [p, p, i32, p, p, i32, p, p, sz, p, p],
            "qmoe_pack_codes": [p, i32, i32, i32, p, p],
            "qmoe_unpack_codes": [p, i32, i32, i32, p, p],
            "qmoe_check_status": [p, p, p],
            "qmoe_status_string": [ctypes.c_int],
            "qmoe_set_dependent_launch": [i32],
            "qmoe_set_prefill_tensor_min": [i32],
            "qmoe_set_decode_wait_limit_ns": [ctypes.c_uint64],
            "qmoe_version": [],
            "qmoe_lfu_create": [i32, p],
            "qmoe_lfu_destroy": [p],
            "qmoe_lfu_plan": [p, p, i32, p, p, p],
            "qmoe_lfu_slots": [p, p, p],
            "qmoe_cache_create": [p, p, p],
            "qmoe_cache_destroy": [p],
            "moe_cache_layer": [p, p, p, i32, p, p, p, p, sz, p, p, p],
            "qmoe_cache_stats": [p, p, p, p, p],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_expert_workspace_bytes.restype = sz
        L.qgemv_affine_workspace_bytes.restype = sz
        L.qgemv_fmt_workspace_bytes.restype = sz
        L.moe_prefill_workspace_bytes.restype = sz
        L.moe_decode_workspace_bytes.restype = sz
        L.moe_decode_pack_bytes.restype = sz
        L.qmoe_status_string.restype = ctypes.c_char_p
        L.qmoe_version.restype = i32
        L.qmoe_set_dependent_launch.restype = i32
        L.qmoe_set_prefill_tensor_min.restype = i32
        L.qmoe_set_decode_wait_limit_ns.restype = ctypes.c_uint64
        L.qmoe_lfu_destroy.restype = None
        L.qmoe_cache_destroy.restype = None
        L.qmoe_lfu_plan.restype = i32
        _lib = L
    return _lib


def status_string(code):
    return lib().qmoe_status_string(int(code)).decode()


def _check(code, what):
    if code != OK:
        raise QmoeError(code, what)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(None)


def _need(t, dtype, what, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % what)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (what, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % what)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (what, tuple(shape), tuple(t.shape)))
    return t


# ----------------------------------------------------------------- weights --
class QMatrix:
    """One affine-quantized matrix (or a stack of `stack` of them) on the GPU.

    packed: int32 [*, rows, cols*bits/32]; scales/biases: float16 [*, rows, cols/64]."""

    def __init__(self, packed, scales, biases, rows, cols, bits, stack=1):
        self.packed, self.scales, self.biases = packed, scales, biases
        self.rows, self.cols, self.bits, self.stack = rows, cols, bits, stack
        _need(packed, torch.int32, "packed")
        _need(scales, torch.float16, "scales")
        _need(biases, torch.float16, "biases")
        if packed.numel() != stack * rows * cols * bits // 32:
            raise ValueError("packed has %d words, expected %d" %
                             (packed.numel(), stack * rows * cols * bits // 32))
        if scales.numel() != stack * rows * cols // 64 or biases.numel() != scales.numel():
            raise ValueError("scales/biases size mismatch")
        self.c = CQMatrix(packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), rows, cols,
                          bits, 64)

    @classmethod
    def from_numpy(cls, P, S, B, rows, cols, bits, device="cuda"):
        """From (packed uint32, scales/biases fp16 bits as uint16) numpy arrays."""
        stack = P.size // (rows * cols * bits // 32)
        packed = torch.from_numpy(P.view("int32").copy()).to(device)
        scales = torch.from_numpy(S.view("float16").copy()).to(device)
        biases = torch.from_numpy(B.view("float16").copy()).to(device)
        return cls(packed, scales, biases, rows, cols, bits, stack)


FMT_ZP4_BF16, FMT_SYM8_BF16 = 1, 2


class CQMatrixFmt(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("params", ctypes.c_void_p),
                ("rht_signs", ctypes.c_void_p), ("rows", ctypes.c_int32),
                ("cols", ctypes.c_int32), ("group", ctypes.c_int32), ("format", ctypes.c_int32)]


class QMatrixFmt:
    """A bf16-scale format-variant matrix on the GPU (zero-point 4-bit or
    symmetric 8-bit), optionally with the block-32 Hadamard rotation signs.

    packed: int32 [rows, cols*bits/32]; params: int32 [rows, cols/64];
    signs: int32 [cols/32] or None."""

    def __init__(self, packed, params, signs, rows, cols, fmt):
        if fmt not in (FMT_ZP4_BF16, FMT_SYM8_BF16):
            raise ValueError("unknown format %r" % (fmt,))
        bits = 4 if fmt == FMT_ZP4_BF16 else 8
        _need(packed, torch.int32, "packed", (rows, cols * bits // 32))
        _need(params, torch.int32, "params", (rows, cols // 64))
        if signs is not None:
            _need(signs, torch.int32, "signs", (cols // 32,))
        self.packed, self.params, self.signs = packed, params, signs
        self.rows, self.cols, self.fmt, self.bits = rows, cols, fmt, bits
        self.c = CQMatrixFmt(packed.data_ptr(), params.data_ptr(),
                             signs.data_ptr() if signs is not None else None, rows, cols, 64, fmt)

    @classmethod
    def from_numpy(cls, P, params, signs, rows, cols, fmt, rotate=True, device="cuda"):
        """From uint32 numpy arrays; `rotate` False drops the rotation."""
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.uint32).view("int32").copy()).to(device)
        return cls(t(P), t(params), t(signs) if rotate else None, rows, cols, fmt)


class MoELayer:
    """Routed experts (stacked gate/up/down) + shared expert (+ optional router)."""

    def __init__(self, gate, up, down, sh_gate, sh_up, sh_down, num_experts, hidden, inter,
                 router=None):
        self.mats = dict(gate=gate, up=up, down=down, sh_gate=sh_gate, sh_up=sh_up,
                         sh_down=sh_down)
        self.router = router
        self.num_experts, self.hidden, self.inter = num_experts, hidden, inter
        self.c = CMoeLayer(gate.c, up.c, down.c, sh_gate.c, sh_up.c, sh_down.c, num_experts,
                           hidden, inter)

    @classmethod
    def from_numpy(cls, m, E, H, I, device="cuda", rank=0, world=1):
        """From a dict like moe_expert_gemv_b200.synth.moe_layer() returns.
        With world > 1, the routed gate/up/down keep only the E/world experts
        rank `rank` holds (for moe_expert_qmlp_ep); shared expert and router
        are whole on every rank."""
        if E % world or not 0 <= rank < world:
            raise ValueError("world must divide E and 0 <= rank < world")
        lo, hi = rank * (E // world), (rank + 1) * (E // world)
        q = {}
        for name, rows, cols in (("gate", I, H), ("up", I, H), ("down", H, I),
                                 ("sh_gate", I, H), ("sh_up", I, H), ("sh_down", H, I)):
            arrs = m[name]
            if world > 1 and not name.startswith("sh_"):
                arrs = tuple(a[lo:hi] for a in arrs)
            q[name] = QMatrix.from_numpy(*arrs, rows, cols, 4, device)
        router = None
        if "router" in m:
            router = QMatrix.from_numpy(*m["router"], E, H, 8, device)
        return cls(q["gate"], q["up"], q["down"], q["sh_gate"], q["sh_up"], q["sh_down"], E, H,
                   I, router)


def expert_owner(e, E, world):
    """Rank that holds expert e when E experts are split over `world` ranks."""
    return e // (E // world)


def moe_expert_qmlp_ep(G, x, idx, weights, rank, world, y_partial=None, workspace=None,
                       status=None):
    """This rank's share of an expert-parallel MoE layer (G from
    MoELayer.from_numpy(..., rank=rank, world=world)): fp32 [H] partial,
    shared expert on rank 0.  The partials of all ranks sum to the layer
    output before its rounding to fp16."""
    x = _need(x, torch.float16, "x")
    top_k = idx.numel()
    if y_partial is None:
        y_partial = torch.empty(G.hidden, dtype=torch.float32, device=x.device)
    _need(y_partial, torch.float32, "y_partial", (G.hidden,))
    ws = workspace if workspace is not None else expert_workspace(G, top_k, x.device)
    _check(lib().moe_expert_qmlp_ep(ctypes.byref(G.c), _ptr(x), _ptr(idx), _ptr(weights), top_k,
                                    rank, world, _ptr(y_partial), _ptr(ws), ws.numel(), _ptr(status),
                                    _stream()), "moe_expert_qmlp_ep")
    return y_partial


def f32_to_f16(src, dst=None):
    """fp32 -> fp16 (round to nearest even) in the library's kernel."""
    src = _need(src, torch.float32, "src")
    if dst is None:
        dst = torch.empty(src.shape, dtype=torch.float16, device=src.device)
    _check(lib().qmoe_f32_to_f16(_ptr(src), _ptr(dst), src.numel(), _stream()), "qmoe_f32_to_f16")
    return dst


def moe_layer_ep(G, x, idx, weights, group=None, workspace=None):
    """One expert-parallel MoE layer on this rank of `group` (torch.distributed,
    NCCL on GPUs): the rank's partial, one all-reduce of the [H] fp32
    partials, then fp16.  Every rank passes the same x, idx and weights (the
    router is replicated)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    yp = moe_expert_qmlp_ep(G, x, idx, weights, rank, world, workspace=workspace)
    dist.all_reduce(yp, group=group)
    return f32_to_f16(yp)


# ------------------------------------------------------- expert streaming --
class LfuPlan:
    """The library's per-layer LFU expert-cache plan alone (host memory only,
    no GPU): step(ids) -> (slot_of [k], [(expert, slot), ...] misses)."""

    def __init__(self, nslots=16):
        h = ctypes.c_void_p()
        _check(lib().qmoe_lfu_create(nslots, ctypes.byref(h)), "qmoe_lfu_create")
        self.h, self.nslots = h, nslots

    def step(self, ids):
        ids = np.ascontiguousarray(ids, np.int32)
        k = ids.size
        slot_of = np.empty(max(k, 1), np.int32)
        me = np.empty(max(k, 1), np.int32)
        ms = np.empty(max(k, 1), np.int32)
        v = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        n = lib().qmoe_lfu_plan(self.h, v(ids), k, v(slot_of), v(me), v(ms))
        if n < 0:
            raise ValueError("k > nslots, k > 16 or repeated ids")
        return slot_of[:k], list(zip(me[:n].tolist(), ms[:n].tolist()))

    def slots(self):
        e = np.empty(self.nslots, np.int32)
        c = np.empty(self.nslots, np.int64)
        _check(lib().qmoe_lfu_slots(self.h, e.ctypes.data_as(ctypes.c_void_p),
                                    c.ctypes.data_as(ctypes.c_void_p)), "qmoe_lfu_slots")
        return e, c

    def __del__(self):
        if getattr(self, "h", None) and _lib is not None:
            _lib.qmoe_lfu_destroy(self.h)
            self.h = None


class ExpertCacheLayer:
    """One MoE layer whose routed experts live in pinned host memory and are
    streamed into `nslots` device slots through the library's LFU plan; the
    router and the shared expert stay on the device."""

    def __init__(self, m, E, H, I, nslots=16, device="cuda"):
        self.E, self.H, self.I, self.nslots = E, H, I, nslots
        pin = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt).copy()).pin_memory()
        self.host = {}
        for name in ("gate", "up", "down"):
            P, S, B = m[name]
            self.host[name] = (pin(P, np.int32), pin(S, np.float16), pin(B, np.float16))
        dims = {"gate": (I, H), "up": (I, H), "down": (H, I)}
        hq = {n: CQMatrix(t[0].data_ptr(), t[1].data_ptr(), t[2].data_ptr(), dims[n][0],
                          dims[n][1], 4, 64) for n, t in self.host.items()}
        dev_layer = MoELayer.from_numpy(m, E, H, I, device)   # router + shared expert on device
        self.router = dev_layer.router
        self.shared = {n: dev_layer.mats[n] for n in ("sh_gate", "sh_up", "sh_down")}
        self.slot = {}
        for n, (rows, cols) in dims.items():
            self.slot[n] = QMatrix(
                torch.zeros(nslots * rows * cols // 8, dtype=torch.int32, device=device),
                torch.zeros(nslots * rows * (cols // 64), dtype=torch.float16, device=device),
                torch.zeros(nslots * rows * (cols // 64), dtype=torch.float16, device=device),
                rows, cols, 4, nslots)
        sh = self.shared
        self.c_host = CMoeLayer(hq["gate"], hq["up"], hq["down"], sh["sh_gate"].c, sh["sh_up"].c,
                                sh["sh_down"].c, E, H, I)
        self.slot_layer = MoELayer(self.slot["gate"], self.slot["up"], self.slot["down"],
                                   sh["sh_gate"], sh["sh_up"], sh["sh_down"], nslots, H, I)
        h = ctypes.c_void_p()
        _check(lib().qmoe_cache_create(ctypes.byref(self.c_host), ctypes.byref(self.slot_layer.c),
                                       ctypes.byref(h)), "qmoe_cache_create")
        self.h = h
        self.workspace = {}
        self.copy_stream = torch.cuda.Stream(device=device)

    def forward(self, x, top_k=8, y=None, idx=None, weights=None, status=None):
        """One decode token x [H] float16 through the layer; returns y [H]."""
        x = _need(x, torch.float16, "x").reshape(-1)
        if y is None:
            y = torch.empty(self.H, dtype=torch.float16, device=x.device)
        ws = self.workspace.get(top_k)
        if ws is None:
            ws = self.workspace[top_k] = expert_workspace(self.slot_layer, top_k, x.device)
        _check(lib().moe_cache_layer(self.h, ctypes.byref(self.router.c), _ptr(x), top_k, _ptr(y),
                                     _ptr(idx), _ptr(weights), _ptr(ws), ws.numel(), _ptr(status),
                                     _stream(), ctypes.c_void_p(self.copy_stream.cuda_stream)),
               "moe_cache_layer")
        return y

    def stats(self):
        """(hits, misses, bytes copied, expert held by each slot)."""
        hits, misses, nbytes = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        slots = np.empty(self.nslots, np.int32)
        _check(lib().qmoe_cache_stats(self.h, ctypes.byref(hits), ctypes.byref(misses),
                                      ctypes.byref(nbytes),
                                      slots.ctypes.data_as(ctypes.c_void_p)), "qmoe_cache_stats")
        return hits.value, misses.value, nbytes.value, slots

    def __del__(self):
        if getattr(self, "h", None) and _lib is not None:
            _lib.qmoe_cache_destroy(self.h)
            self.h = None


# ------------------------------------------------------------- operations --
# zero-filled workspace of qgemv_affine_ws, one per device (allocated by the
# first call that needs it, so a CUDA graph captured after a first call
# reuses it); calls that can run at the same time on different streams must
# pass their own workspace
_qgemv_ws = {}


def qgemv_workspace(W, batch, device=None):
    """A zero-filled workspace for qgemv_affine_ws calls on W at this batch
    (None when none is needed)."""
    need = lib().qgemv_affine_workspace_bytes(W.rows, W.cols, W.bits, batch)
    if not need:
        return None
    return torch.zeros(need, dtype=torch.uint8, device=device or torch.device("cuda"))


def _shared_workspace(nbytes, device):
    ws = _qgemv_ws.get(device.index)
    if ws is None or ws.numel() < nbytes:
        if torch.cuda.is_current_stream_capturing():
            raise RuntimeError("qgemv_affine: no workspace of %d bytes yet on this device; call it "
                               "once before capturing, or pass workspace=" % nbytes)
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _qgemv_ws[device.index] = ws
    return ws


def qgemv_affine(W, x, y=None, status=None, one_pass=True, workspace=None):
    """y[b] = W x[b] for x [B][K] float16 (B <= 32).  Returns y [B][N] float16.
    A batch of 9..32 runs in one pass over the weights (qgemv_affine_ws) where
    the shape allows it, with `workspace` (a zero-filled uint8 tensor, see
    qgemv_workspace) or else one kept per device; one_pass=False runs one
    qGEMV launch per 8 rows (qgemv_affine)."""
    x = _need(x, torch.float16, "x")
    x2 = x.reshape(-1, W.cols)
    B = x2.shape[0]
    if y is None:
        y = torch.empty(B, W.rows, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", (B, W.rows))
    need = lib().qgemv_affine_workspace_bytes(W.rows, W.cols, W.bits, B) if one_pass and B > 8 else 0
    if need:
        ws = workspace if workspace is not None else _shared_workspace(need, x.device)
        _check(lib().qgemv_affine_ws(ctypes.byref(W.c), _ptr(x2), B, _ptr(y), _ptr(ws),
                                     ws.numel() * ws.element_size(), _ptr(status), _stream()),
               "qgemv_affine_ws")
    else:
        _check(lib().qgemv_affine(ctypes.byref(W.c), _ptr(x2), B, _ptr(y), _ptr(status),
                                  _stream()), "qgemv_affine")
    return y


def qgemv_fmt(W, x, y=None, status=None, one_pass=True, workspace=None):
    """y[b] = W (R x[b]) (R the rotation when W has signs) for x [B][K]
    float16 (B <= 32), W a QMatrixFmt.  Returns y [B][N] float16.  A batch
    of 9..32 runs in one pass over the weights (qgemv_fmt_ws) where the shape
    allows it (workspace as qgemv_affine); one_pass=False runs one launch per
    8 rows."""
    x = _need(x, torch.float16, "x")
    x2 = x.reshape(-1, W.cols)
    B = x2.shape[0]
    if y is None:
        y = torch.empty(B, W.rows, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", (B, W.rows))
    rotated = 1 if W.c.rht_signs else 0
    need = (lib().qgemv_fmt_workspace_bytes(W.rows, W.cols, W.c.format, rotated, B)
            if one_pass and B > 8 else 0)
    if one_pass and B > 8:
        ws = None
        if need:
            ws = workspace if workspace is not None else _shared_workspace(need, x.device)
        _check(lib().qgemv_fmt_ws(ctypes.byref(W.c), _ptr(x2), B, _ptr(y), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(),
                                  _ptr(status), _stream()), "qgemv_fmt_ws")
    else:
        _check(lib().qgemv_fmt(ctypes.byref(W.c), _ptr(x2), B, _ptr(y), _ptr(status), _stream()),
               "qgemv_fmt")
    return y


def moe_router_topk(router, x, top_k, idx=None, weights=None, logits=None, want_logits=False,
                    status=None):
    """Router logits -> softmax -> top-k -> renormalised weights for x [T][K].
    Returns (idx int32 [T][k], weights float32 [T][k], logits float32 [T][E] or None)."""
    x = _need(x, torch.float16, "x")
    x2 = x.reshape(-1, router.cols)
    T = x2.shape[0]
    dev = x.device
    if idx is None:
        idx = torch.empty(T, top_k, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(T, top_k, dtype=torch.float32, device=dev)
    if logits is None and want_logits:
        logits = torch.empty(T, router.rows, dtype=torch.float32, device=dev)
    _need(idx, torch.int32, "idx", (T, top_k))
    _need(weights, torch.float32, "weights", (T, top_k))
    if logits is not None:
        _need(logits, torch.float32, "logits", (T, router.rows))
    _check(lib().moe_router_topk(ctypes.byref(router.c), _ptr(x2), T, top_k, _ptr(idx),
                                 _ptr(weights), _ptr(logits), _ptr(status), _stream()),
           "moe_router_topk")
    return idx, weights, logits


def moe_expert_workspace_bytes(layer, top_k):
    return lib().moe_expert_workspace_bytes(ctypes.byref(layer.c), top_k)


def expert_workspace(layer, top_k, device="cuda"):
    """A zero-filled workspace for moe_expert_qmlp (reusable across calls)."""
    n = moe_expert_workspace_bytes(layer, top_k)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_expert_qmlp(layer, x, idx, weights, y=None, workspace=None, status=None):
    """y = shared(x) + sum_j weights[j] * expert_{idx[j]}(x) for one token x [H]."""
    x = _need(x, torch.float16, "x").reshape(-1)
    top_k = idx.numel()
    _need(idx, torch.int32, "idx")
    _need(weights, torch.float32, "weights")
    if y is None:
        y = torch.empty(layer.hidden, dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = expert_workspace(layer, top_k, x.device)
    _check(lib().moe_expert_qmlp(ctypes.byref(layer.c), _ptr(x), _ptr(idx), _ptr(weights), top_k,
                                 _ptr(y), _ptr(workspace), workspace.numel(), _ptr(status),
                                 _stream()), "moe_expert_qmlp")
    return y


def moe_expert_gateup(layer, x, idx, workspace, status=None):
    x = _need(x, torch.float16, "x").reshape(-1)
    _check(lib().moe_expert_gateup(ctypes.byref(layer.c), _ptr(x), _ptr(idx), idx.numel(),
                                   _ptr(workspace), workspace.numel(), _ptr(status), _stream()),
           "moe_expert_gateup")


def moe_expert_down(layer, idx, weights, y, workspace, status=None):
    _check(lib().moe_expert_down(ctypes.byref(layer.c), _ptr(idx), _ptr(weights), idx.numel(),
                                 _ptr(y), _ptr(workspace), workspace.numel(), _ptr(status),
                                 _stream()), "moe_expert_down")
    return y


class DecodeStack:
    """A stack of MoE layers (each with its router) repacked once into the
    fused decode kernel's streaming layout, plus its zero-filled workspace."""

    def __init__(self, layers, top_k, device="cuda"):
        self.layers = list(layers)
        L0 = self.layers[0]
        self.top_k = top_k
        self.E, self.H, self.I = L0.num_experts, L0.hidden, L0.inter
        nbytes = lib().moe_decode_pack_bytes(ctypes.byref(L0.c))
        if nbytes == 0:
            raise ValueError("layer shape not supported by the fused decode")
        self.packed = []
        for L in self.layers:
            buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
            _check(lib().moe_decode_pack_layer(ctypes.byref(L.c), ctypes.byref(L.router.c),
                                               _ptr(buf), nbytes, _stream()),
                   "moe_decode_pack_layer")
            self.packed.append(buf)
        torch.cuda.current_stream().synchronize()
        self.c_packed = (ctypes.c_void_p * len(self.packed))(*[b.data_ptr() for b in self.packed])
        ws = lib().moe_decode_workspace_bytes(self.E, self.H, self.I, top_k)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)


def moe_decode_layers(stack, x, y=None, idx=None, weights=None, logits=None, status=None):
    """One token per layer through the whole stack in one fused launch.
    x, y: float16 [n_layers][hidden]; idx int32 / weights float32 [n_layers][top_k];
    logits float32 [n_layers][num_experts] (optional)."""
    n = len(stack.packed)
    x = _need(x, torch.float16, "x", (n, stack.H))
    if y is None:
        y = torch.empty(n, stack.H, dtype=torch.float16, device=x.device)
    _need(y, torch.float16, "y", (n, stack.H))
    if idx is not None:
        _need(idx, torch.int32, "idx", (n, stack.top_k))
    if weights is not None:
        _need(weights, torch.float32, "weights", (n, stack.top_k))
    if logits is not None:
        _need(logits, torch.float32, "logits", (n, stack.E))
    _check(lib().moe_decode_layers(stack.c_packed, n, stack.E, stack.H, stack.I, _ptr(x),
                                   stack.top_k, _ptr(y), _ptr(idx), _ptr(weights), _ptr(logits),
                                   _ptr(stack.workspace), stack.workspace.numel(), _ptr(status),
                                   _stream()), "moe_decode_layers")
    return y


def moe_decode_layers_host(stack, x_host, y_host, x_dev, y_dev, status=None):
    """The decode step from host buffers through the C call that copies them:
    x_host -> x_dev, the fused decode, y_dev -> y_host, enqueued on the
    current stream (synchronise before reading y_host).  x_host / y_host:
    float16 [n_layers][hidden] CPU tensors (pinned for asynchronous copies);
    x_dev / y_dev: device staging tensors of the same shape."""
    n = len(stack.packed)
    for t, name in ((x_host, "x_host"), (y_host, "y_host")):
        if t.device.type != "cpu" or t.dtype != torch.float16 or tuple(t.shape) != (n, stack.H) \
                or not t.is_contiguous():
            raise ValueError("%s: expected a contiguous CPU float16 [%d, %d] tensor" % (name, n, stack.H))
    _need(x_dev, torch.float16, "x_dev", (n, stack.H))
    _need(y_dev, torch.float16, "y_dev", (n, stack.H))
    _check(lib().moe_decode_layers_host(stack.c_packed, n, stack.E, stack.H, stack.I,
                                        ctypes.c_void_p(x_host.data_ptr()),
                                        ctypes.c_void_p(y_host.data_ptr()), stack.top_k,
                                        _ptr(x_dev), _ptr(y_dev), _ptr(stack.workspace),
                                        stack.workspace.numel(), _ptr(status), _stream()),
           "moe_decode_layers_host")
    return y_host


def moe_group_tokens(idx, num_experts, status=None):
    """Counting sort of a chunk's (token, slot) pairs by expert.
    Returns (counts [E], offsets [E+1], pairs [T*k]) int32."""
    _need(idx, torch.int32, "idx")
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(num_experts, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    pairs = torch.empty(T * k, dtype=torch.int32, device=dev)
    _check(lib().moe_group_tokens(_ptr(idx), T, k, num_experts, _ptr(counts), _ptr(offsets),
                                  _ptr(pairs), _ptr(status), _stream()), "moe_group_tokens")
    return counts, offsets, pairs


def moe_prefill_workspace_bytes(layer, tokens, top_k):
    return lib().moe_prefill_workspace_bytes(ctypes.byref(layer.c), tokens, top_k)


def moe_prefill_qgemm(layer, x, idx, weights, y=None, workspace=None, status=None):
    """y[t] = shared(x[t]) + sum_j weights[t][j] expert_{idx[t][j]}(x[t]), x [T][H]."""
    x = _need(x, torch.float16, "x")
    T = x.shape[0]
    _need(idx, torch.int32, "idx")
    _need(weights, torch.float32, "weights")
    top_k = idx.shape[1]
    if y is None:
        y = torch.empty(T, layer.hidden, dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = torch.empty(moe_prefill_workspace_bytes(layer, T, top_k), dtype=torch.uint8,
                                device=x.device)
    _check(lib().moe_prefill_qgemm(ctypes.byref(layer.c), _ptr(x), T, _ptr(idx), _ptr(weights),
                                   top_k, _ptr(y), _ptr(workspace), workspace.numel(),
                                   _ptr(status), _stream()), "moe_prefill_qgemm")
    return y


def qmoe_pack_codes(codes, bits):
    """uint8 codes [rows][cols] -> int32 packed words [rows][cols*bits/32]."""
    _need(codes, torch.uint8, "codes")
    rows, cols = codes.shape
    packed = torch.empty(rows, cols * bits // 32, dtype=torch.int32, device=codes.device)
    _check(lib().qmoe_pack_codes(_ptr(codes), rows, cols, bits, _ptr(packed), _stream()),
           "qmoe_pack_codes")
    return packed


def qmoe_unpack_codes(packed, rows, cols, bits):
    _need(packed, torch.int32, "packed")
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=packed.device)
    _check(lib().qmoe_unpack_codes(_ptr(packed), rows, cols, bits, _ptr(codes), _stream()),
           "qmoe_unpack_codes")
    return codes


def qmoe_check_status(status=None):
    """Synchronise the current stream; return the device flags (and clear them).
    Raises QmoeError on a CUDA failure; flags are returned, not raised."""
    flags = ctypes.c_int32(0)
    rc = lib().qmoe_check_status(_ptr(status), _stream(), ctypes.byref(flags))
    if rc not in (OK, -5, -6):
        raise QmoeError(rc, "qmoe_check_status")
    return flags.value


def qmoe_set_dependent_launch(enable):
    return bool(lib().qmoe_set_dependent_launch(1 if enable else 0))


def qmoe_set_decode_wait_limit_ns(ns):
    """Limit of every wait inside the fused decode (0: the default 2 s).
    Returns the previous setting."""
    return int(lib().qmoe_set_decode_wait_limit_ns(int(ns)))


# the threshold used when the tensor-core prefill path is switched on (the
# library's own default is 0: off)
TENSOR_MIN_DEFAULT = 16


def qmoe_set_prefill_tensor_min(min_tokens):
    """Experts of a prefill chunk with at least min_tokens tokens run on the
    tensor-core kernels (0: none).  Returns the previous setting."""
    return int(lib().qmoe_set_prefill_tensor_min(int(min_tokens)))


def qmoe_version():
    return lib().qmoe_version()
