"""Seeded synthetic inputs shaped like the workloads the pages describe.

This module draws random numbers and lays them out in the packed storage
format; it holds none of the method's arithmetic (no dequantisation, no
products, no routing).  Both the CPU oracle (through the tests) and the CUDA
library consume exactly the arrays it returns.

Recipe (every tensor has its own stream, seeded from (seed, layer, tensor)):
  * codes q: uniform over [0, 2^bits); because every code value is equally
    likely and codes are independent, a packed word of uniform codes is a
    uniform random 32-bit word, so the packed words are drawn directly;
  * scales / biases: drawn in fp64 from the stated uniform ranges, then
    rounded to fp16 (round to nearest even);
  * activations x: N(0, 1) drawn in fp64, rounded to fp16;
  * prefill routing: expert ranks r = 1..E with P(r) proportional to r^-s
    (Zipf, s = 1.1); a seeded permutation maps ranks to expert ids; each token
    draws top_k distinct experts by the Gumbel-top-k trick on log P(r), which
    is sampling without replacement; the combine weights are positive draws
    U(0.05, 1) normalised to sum to one and listed in descending order.

Shapes follow the TurboFieldfare article (jeff.news): MLX affine 4-bit group-64
experts, an 8-bit router, top-8 routing, prefill chunks of 128 tokens.
fp16 tensors are returned as uint16 bit patterns.
"""
import numpy as np

# tensor tags for the seed streams
_TAGS = {"x": 1, "router": 2, "gate": 3, "up": 4, "down": 5, "sh_gate": 6, "sh_up": 7,
         "sh_down": 8, "dense": 9, "assign": 10, "weights": 11, "perm": 12}

# value ranges
DENSE_SCALE = (0.005, 0.02)
DENSE_BIAS = (-0.1, 0.1)
ROUTER_SCALE = (0.001, 0.004)
ROUTER_BIAS = (-0.2, 0.2)

# the MoE layer of the decode / prefill workloads
MOE_E, MOE_H, MOE_I, MOE_TOPK, MOE_LAYERS = 128, 2816, 704, 8, 30
PREFILL_T, ZIPF_S = 128, 1.1


def rng(seed, *tags):
    return np.random.default_rng(np.random.SeedSequence([int(seed)] + [int(t) for t in tags]))


def to_f16_bits(a):
    return np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def random_words(g, shape):
    n = int(np.prod(shape))
    return np.frombuffer(g.bytes(4 * n), dtype=np.uint32).reshape(shape).copy()


def qmatrix(g, rows, cols, bits=4, scale=DENSE_SCALE, bias=DENSE_BIAS, lead=()):
    """(packed uint32 [*lead, rows, cols*bits/32], scales u16 [*lead, rows, cols/64],
    biases u16 [...]) with uniform codes."""
    assert cols % 64 == 0 and bits in (4, 8)
    lead = tuple(lead)
    P = random_words(g, lead + (rows, cols * bits // 32))
    S = to_f16_bits(g.uniform(scale[0], scale[1], lead + (rows, cols // 64)))
    B = to_f16_bits(g.uniform(bias[0], bias[1], lead + (rows, cols // 64)))
    return P, S, B


FMT_ZP4, FMT_SYM8 = 1, 2
SYM8_SCALE = (0.001, 0.004)


def to_bf16_bits(a):
    """fp64 values -> bf16 bit patterns (via fp32, round to nearest even)."""
    u = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def qmatrix_fmt(g, rows, cols, fmt):
    """Format-variant matrix: (packed uint32 [rows][cols*bits/32], params uint32
    [rows][cols/64] = bf16 scale | zero point << 16, signs uint32 [cols/32]).
    ZP4: 4-bit codes, zero points uniform in 0..15, scales U(0.005, 0.02);
    SYM8: 8-bit two's-complement codes, scales U(0.001, 0.004)."""
    assert cols % 64 == 0 and fmt in (FMT_ZP4, FMT_SYM8)
    bits = 4 if fmt == FMT_ZP4 else 8
    P = random_words(g, (rows, cols * bits // 32))
    lo, hi = DENSE_SCALE if fmt == FMT_ZP4 else SYM8_SCALE
    S = to_bf16_bits(g.uniform(lo, hi, (rows, cols // 64))).astype(np.uint32)
    Z = (g.integers(0, 16, (rows, cols // 64)).astype(np.uint32) if fmt == FMT_ZP4
         else np.zeros((rows, cols // 64), np.uint32))
    signs = random_words(g, (cols // 32,))
    return P, S | (Z << 16), signs


def activations(seed, rows, cols, layer=0):
    """x [rows][cols] ~ N(0,1), fp16 bits."""
    return to_f16_bits(rng(seed, layer, _TAGS["x"]).standard_normal((rows, cols)))


def correlated_tokens(seed, T, cols, rho, layer=0):
    """fp16 bits [T][cols]: x_0 ~ N(0,1), x_t = rho x_{t-1} + sqrt(1 - rho^2) n_t
    (each row stays N(0,1)); rho near 1 gives consecutive tokens similar
    routing, rho = 0 independent tokens."""
    g = rng(seed, layer, 17)
    x = np.empty((T, cols))
    x[0] = g.standard_normal(cols)
    for t in range(1, T):
        x[t] = rho * x[t - 1] + np.sqrt(1.0 - rho * rho) * g.standard_normal(cols)
    return to_f16_bits(x)


def dense(seed, N, K, bits=4, layer=0):
    """One dense affine-quantized matrix with the dense-GEMV value ranges."""
    return qmatrix(rng(seed, layer, _TAGS["dense"]), N, K, bits)


def router(seed, E=MOE_E, K=MOE_H, layer=0):
    """The 8-bit router [E][K] with the router value ranges."""
    return qmatrix(rng(seed, layer, _TAGS["router"]), E, K, 8, ROUTER_SCALE, ROUTER_BIAS)


def moe_layer(seed, layer=0, E=MOE_E, H=MOE_H, I=MOE_I, bits=4, with_router=True):
    """Dict of (packed, scales, biases) for gate/up [E][I][H], down [E][H][I],
    sh_gate/sh_up [I][H], sh_down [H][I] and router [E][H] (8-bit)."""
    m = {}
    for name, rows, cols, lead in (("gate", I, H, (E,)), ("up", I, H, (E,)),
                                   ("down", H, I, (E,)), ("sh_gate", I, H, ()),
                                   ("sh_up", I, H, ()), ("sh_down", H, I, ())):
        m[name] = qmatrix(rng(seed, layer, _TAGS[name]), rows, cols, bits, lead=lead)
    if with_router:
        m["router"] = router(seed, E, H, layer)
    return m


def zipf_routing(seed, T=PREFILL_T, E=MOE_E, k=MOE_TOPK, s=ZIPF_S):
    """(idx [T][k] int32 distinct experts per token, wt [T][k] fp32 descending,
    summing to one)."""
    g = rng(seed, 0, _TAGS["assign"])
    logp = -s * np.log(np.arange(1, E + 1, dtype=np.float64))
    perm = rng(seed, 0, _TAGS["perm"]).permutation(E)
    keys = logp[None, :] + g.gumbel(size=(T, E))
    ranks = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    idx = perm[ranks].astype(np.int32)
    u = rng(seed, 0, _TAGS["weights"]).uniform(0.05, 1.0, (T, k))
    u = -np.sort(-u, axis=1)
    wt = (u / u.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, wt
