"""Seeded synthetic inputs for the routed-expert MoE layer.

This module is the only code shared between the CPU oracle (``oracle/``) and
the CUDA path: it produces *inputs* (activations, router logits, MXFP4 expert
weights, random FP8 operands) and holds none of the arithmetic of the layer
itself.  Everything is generated on the host with numpy from a counter-based
generator, so both sides see identical bytes.

Generator: splitmix64 (S. Vigna's published mixing function) used in counter
mode -- output ``i`` of stream ``s`` under ``seed`` is
``mix(key(seed, s) + (i + 1) * 0x9E3779B97F4A7C15)``; each tensor draws from
its own stream so tensors do not depend on generation order.  Normals use the
Box-Muller transform.

The workload recipes follow the shapes of a DeepSeek-V4-Flash-class MoE layer
(hidden 4096, expert intermediate 2048, 256 routed + 1 shared experts, top-6),
as given on the "DeepSeek-V4-Flash-SI" model card (section 模型概述 and the
MoE paragraph of 架构特性).
"""
from __future__ import annotations

import dataclasses

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser, in place on a uint64 array (returns it)."""
    t = np.empty_like(z)
    np.right_shift(z, np.uint64(30), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, _M1, out=z)
    np.right_shift(z, np.uint64(27), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, _M2, out=z)
    np.right_shift(z, np.uint64(31), out=t)
    np.bitwise_xor(z, t, out=z)
    return z


def _key(seed: int, stream: int) -> np.uint64:
    if not (seed or stream):
        return np.uint64(0)
    with np.errstate(over="ignore"):
        return _mix(np.array([(seed * 0x632BE59BD9B4E019 + stream) & 0xFFFFFFFFFFFFFFFF],
                             dtype=np.uint64))[0]


_STEP = 1 << 20


def _parallel(n: int, fn) -> None:
    """Run fn(i0, i1) over chunks of [0, n); numpy ufuncs release the GIL, so
    chunks run on several host cores.  Results do not depend on the split."""
    chunks = [(i0, min(n, i0 + _STEP)) for i0 in range(0, n, _STEP)]
    if len(chunks) <= 2:
        for c in chunks:
            fn(*c)
        return
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda c: fn(*c), chunks))


def _stream_values(key: np.uint64, c0: int, c1: int) -> np.ndarray:
    """Outputs c0 .. c1-1 (0-based) of the stream with the given key."""
    with np.errstate(over="ignore"):
        z = np.arange(c0 + 1, c1 + 1, dtype=np.uint64)
        np.multiply(z, _GAMMA, out=z)
        np.add(z, key, out=z)
        return _mix(z)


def splitmix64(seed: int, stream: int, n: int) -> np.ndarray:
    """n uint64 outputs of the counter-mode splitmix64 stream (seed, stream)."""
    key = _key(seed, stream)
    out = np.empty(n, np.uint64)

    def work(i0, i1):
        out[i0:i1] = _stream_values(key, i0, i1)

    _parallel(n, work)
    return out


def uniform(seed: int, stream: int, n: int) -> np.ndarray:
    """n doubles in [0, 1) with 53 random bits each."""
    return (splitmix64(seed, stream, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normals (Box-Muller, cosine branch): normal i uses stream
    outputs 2i (radius) and 2i+1 (angle)."""
    key = _key(seed, stream)
    out = np.empty(n, np.float64)

    def work(i0, i1):
        u = (_stream_values(key, 2 * i0, 2 * i1) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        out[i0:i1] = np.sqrt(-2.0 * np.log1p(-u[0::2])) * np.cos(2.0 * np.pi * u[1::2])

    _parallel(n, work)
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bfloat16 (round to nearest even), as uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# MXFP4 weight synthesis (an input format, not a step of the layer).
# Each block of 32 values gets the exponent e = ceil(log2(amax / 6)) so the
# block maximum lands in (3, 6]; values are rounded to the nearest E2M1 grid
# point with ties to the even code, saturating at 6.  All-zero blocks get e=0.
# ---------------------------------------------------------------------------
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _round_to_e2m1_code(m: np.ndarray) -> np.ndarray:
    """Magnitudes (already divided by the block scale) -> 3-bit codes 0..7,
    nearest grid point, ties to the even code, saturating at 6."""
    mid = (_E2M1_GRID[1:] + _E2M1_GRID[:-1]) / 2          # 0.25, 0.75, ..., 5
    c = np.searchsorted(mid, m, side="left")              # number of midpoints below m
    tie = (c < 7) & (m == mid[np.minimum(c, 6)]) & (c % 2 == 1)
    return (c + tie).astype(np.uint8)


def quantize_mxfp4(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Row-parallel wrapper of _quantize_mxfp4 (same result for any split)."""
    w = np.asarray(w, dtype=np.float64)
    if w.ndim != 2 or w.shape[0] < 64:
        return _quantize_mxfp4(w)
    rows = w.shape[0]
    packed = np.empty((rows, w.shape[1] // 2), np.uint8)
    scales = np.empty((rows, w.shape[1] // 32), np.uint8)
    step = max(1, (1 << 18) // w.shape[1])

    def work(r0, r1):
        for a in range(r0, r1, step):
            b = min(r1, a + step)
            packed[a:b], scales[a:b] = _quantize_mxfp4(w[a:b])

    import concurrent.futures as cf
    import os
    n = min(16, os.cpu_count() or 1)
    bounds = [(rows * i // n, rows * (i + 1) // n) for i in range(n)]
    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(lambda c: work(*c), bounds))
    return packed, scales


def _quantize_mxfp4(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """float [..., K] -> (packed nibbles uint8 [..., K/2], E8M0 uint8 [..., K/32]).

    Element 2i sits in the low nibble, 2i+1 in the high nibble.
    """
    w = np.asarray(w, dtype=np.float64)
    K = w.shape[-1]
    assert K % 32 == 0
    blocks = w.reshape(*w.shape[:-1], K // 32, 32)
    amax = np.abs(blocks).max(axis=-1)
    with np.errstate(divide="ignore"):
        ratio = amax / 6.0
        e = np.where(amax > 0, np.ceil(np.log2(np.where(amax > 0, ratio, 1.0))), 0.0)
    # (the code below keeps every step vectorised; memory stays O(size))
    # guard against log2 rounding: make sure amax / 2^e <= 6 and > 3
    e = np.where((amax > 0) & (amax / np.exp2(e) > 6.0), e + 1, e)
    e = np.where((amax > 0) & (amax / np.exp2(e) <= 3.0), e - 1, e)
    e = np.clip(e, -127, 127)
    scaled = blocks / np.exp2(e)[..., None]
    code = _round_to_e2m1_code(np.abs(scaled))
    sign = ((scaled < 0) & (code > 0)).astype(np.uint8)
    nib = (code | (sign << 3)).reshape(*w.shape[:-1], K)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return packed, (e + 127).astype(np.uint8)


# ---------------------------------------------------------------------------
# Layer workloads
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class MoeWorkload:
    name: str
    T: int
    H: int
    I: int
    E: int
    topk: int
    x_bf16: np.ndarray          # uint16 [T, H]
    logits: np.ndarray          # float32 [T, E]
    w13: np.ndarray             # uint8 [E+1, 2I, H/2]  (w1 = gate rows, then w3 = up rows)
    w13_e8m0: np.ndarray        # uint8 [E+1, 2I, H/32]
    w2: np.ndarray              # uint8 [E+1, H, I/2]
    w2_e8m0: np.ndarray         # uint8 [E+1, H, I/32]
    route_scale: float = 1.5
    swiglu_limit: float = 10.0


class RepeatedExperts:
    """Read-only [E1, ...] view of per-expert arrays in which expert e holds
    prototype e % n (the n_proto recipe of expert_weights) without copying:
    indexing by an expert gives its prototype, a slice gives a stacked copy,
    materialize() the whole array."""

    def __init__(self, protos: np.ndarray, E1: int):
        self.protos = protos
        self.shape = (E1,) + protos.shape[1:]
        self.dtype = protos.dtype
        self.ndim = len(self.shape)

    def __len__(self):
        return self.shape[0]

    def __getitem__(self, g):
        n = len(self.protos)
        if isinstance(g, (int, np.integer)):
            if not -self.shape[0] <= g < self.shape[0]:
                raise IndexError(g)
            return self.protos[int(g) % self.shape[0] % n]
        if isinstance(g, slice):
            return self.protos[np.arange(self.shape[0])[g] % n]
        raise TypeError("index an expert by int or slice")

    def materialize(self) -> np.ndarray:
        return self.protos[np.arange(self.shape[0]) % len(self.protos)]


def expert_prototypes(seed: int, n: int, H: int, I: int, std: float = 0.02):
    """The first n experts of expert_weights: MXFP4 w13 [n, 2I, H/2] + E8M0,
    w2 [n, H, I/2] + E8M0, expert e from its own streams."""
    w13 = np.empty((n, 2 * I, H // 2), np.uint8)
    s13 = np.empty((n, 2 * I, H // 32), np.uint8)
    w2 = np.empty((n, H, I // 2), np.uint8)
    s2 = np.empty((n, H, I // 32), np.uint8)
    for e in range(n):
        a = normal(seed, 1000 + 2 * e, 2 * I * H).reshape(2 * I, H) * std
        w13[e], s13[e] = quantize_mxfp4(a)
        b = normal(seed, 1001 + 2 * e, H * I).reshape(H, I) * std
        w2[e], s2[e] = quantize_mxfp4(b)
    return w13, s13, w2, s2


def expert_views(seed: int, E1: int, H: int, I: int, n_proto: int, std: float = 0.02):
    """expert_weights(seed, E1, H, I, std, n_proto) as RepeatedExperts views
    (the same values, drawn once per prototype, nothing repeated in memory)."""
    protos = expert_prototypes(seed, min(E1, n_proto), H, I, std)
    return tuple(RepeatedExperts(p, E1) for p in protos)


def expert_weights(seed: int, E1: int, H: int, I: int, std: float = 0.02, n_proto: int | None = None):
    """MXFP4 w13 [E1, 2I, H] (w1 rows then w3 rows) and w2 [E1, H, I] from N(0, std).

    Expert e draws from its own streams.  With ``n_proto`` set, only the first
    n_proto experts are drawn and expert e repeats expert e % n_proto (distinct
    memory, same values): full-size layers then take seconds to synthesise
    while every expert still streams its own bytes."""
    n_draw = E1 if n_proto is None else min(E1, n_proto)
    protos = expert_prototypes(seed, n_draw, H, I, std)
    if n_draw == E1:
        return protos
    return tuple(RepeatedExperts(p, E1).materialize() for p in protos)


def tiny_layer(seed: int = 0) -> MoeWorkload:
    """Hidden 256, intermediate 128, 8 routed + 1 shared, top-2, 16 tokens.

    Router logits = x . Wg^T with Wg ~ N(0, 0.02), computed on the host (the
    gate projection is not part of the expert path)."""
    T, H, I, E, k = 16, 256, 128, 8, 2
    x = to_bf16_bits(normal(seed, 1, T * H).reshape(T, H))
    wg = normal(seed, 2, E * H).reshape(E, H) * 0.02
    logits = (bf16_bits_to_f32(x).astype(np.float64) @ wg.T).astype(np.float32)
    w13, s13, w2, s2 = expert_weights(seed, E + 1, H, I)
    return MoeWorkload("tiny", T, H, I, E, k, x, logits, w13, s13, w2, s2)


def _values_at(key: np.uint64, counters: np.ndarray) -> np.ndarray:
    """Outputs at the given 0-based counters of the stream with this key."""
    with np.errstate(over="ignore"):
        z = np.asarray(counters, dtype=np.uint64) + np.uint64(1)
        np.multiply(z, _GAMMA, out=z)
        np.add(z, key, out=z)
        return _mix(z)


def decode_activations(seed: int, T: int, H: int, rows=None) -> np.ndarray:
    """N(0,1) with each element scaled x20 with probability 0.001 (outliers).

    rows: optional token indices; then only those rows of the [T, H] batch
    are generated (the same values, from the same counters)."""
    if rows is None:
        x = normal(seed, 1, T * H)
        out = uniform(seed, 3, T * H) < 0.001
        x = np.where(out, 20.0 * x, x)
        return to_bf16_bits(x.reshape(T, H))
    rows = np.asarray(rows, dtype=np.int64)
    i = (rows[:, None] * H + np.arange(H)[None, :]).reshape(-1)
    k1 = _key(seed, 1)
    u1 = (_values_at(k1, 2 * i) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    u2 = (_values_at(k1, 2 * i + 1) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    x = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)
    out = (_values_at(_key(seed, 3), i) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53) < 0.001
    x = np.where(out, 20.0 * x, x)
    return to_bf16_bits(x.reshape(len(rows), H))


def uniform_logits(seed: int, T: int, E: int) -> np.ndarray:
    return (uniform(seed, 4, T * E) * 2.0 - 1.0).astype(np.float32).reshape(T, E)


def zipf_logits(seed: int, T: int, E: int, s: float = 1.1) -> np.ndarray:
    """log p_e + Gumbel(0,1) noise with p_e proportional to rank^-s.

    Top-k of Gumbel-perturbed log-probabilities draws experts without
    replacement with probabilities p, so expert loads follow the Zipf law
    (flattened at the head because each token picks k distinct experts).
    Expert e has rank e+1."""
    logp = -s * np.log(np.arange(1, E + 1, dtype=np.float64))
    logp -= np.log(np.exp(logp).sum())
    u = uniform(seed, 5, T * E).reshape(T, E)
    g = -np.log(-np.log(np.clip(u, 1e-300, None)))
    return (logp[None, :] + g).astype(np.float32)


def random_e4m3(seed: int, stream: int, shape, max_code: int = 0x7E) -> np.ndarray:
    """Random finite E4M3 bytes (codes 0x7F / 0xFF are NaN and never drawn)."""
    n = int(np.prod(shape))
    r = splitmix64(seed, stream, n)
    mag = (r % np.uint64(max_code + 1)).astype(np.uint8)
    sign = ((r >> np.uint64(32)) & np.uint64(1)).astype(np.uint8) << 7
    return (mag | sign).reshape(shape)


def random_bytes(seed: int, stream: int, shape, lo: int = 0, hi: int = 255) -> np.ndarray:
    n = int(np.prod(shape))
    r = splitmix64(seed, stream, n)
    return (lo + (r % np.uint64(hi - lo + 1))).astype(np.uint8).reshape(shape)


def small_int_e4m3(seed: int, stream: int, shape) -> np.ndarray:
    """E4M3 codes of the integers -4..4 (exact products with E2M1 integers)."""
    table = np.array([0xC8, 0xC4, 0xC0, 0xB8, 0x00, 0x38, 0x40, 0x44, 0x48], np.uint8)
    n = int(np.prod(shape))
    return table[(splitmix64(seed, stream, n) % np.uint64(9)).astype(np.int64)].reshape(shape)


def small_int_fp4(seed: int, stream: int, shape_packed) -> np.ndarray:
    """Packed E2M1 bytes whose nibbles are the integer codes 0,+-1,+-2,+-3,+-4,+-6."""
    codes = np.array([0x0, 0x2, 0x4, 0x5, 0x6, 0x7, 0xA, 0xC, 0xD, 0xE, 0xF], np.uint8)
    n = int(np.prod(shape_packed))
    r = splitmix64(seed, stream, n)
    lo = codes[(r % np.uint64(11)).astype(np.int64)]
    hi = codes[((r >> np.uint64(8)) % np.uint64(11)).astype(np.int64)]
    return (lo | (hi << 4)).astype(np.uint8).reshape(shape_packed)


def hash_table(seed: int, vocab: int, E: int, k: int) -> np.ndarray:
    """A token-id -> expert table int32 [vocab, k]: k distinct expert ids per
    entry, drawn uniformly without replacement (a partial Fisher-Yates shuffle
    of 0..E-1 per entry, one 64-bit draw per swap).  It stands in for the
    table a checkpoint carries for the hash-routed layers."""
    assert 1 <= k <= E
    r = splitmix64(seed, 6, vocab * k).reshape(vocab, k)
    perm = np.tile(np.arange(E, dtype=np.int64), (vocab, 1))
    rows = np.arange(vocab)
    for j in range(k):
        pick = j + (r[:, j] % np.uint64(E - j)).astype(np.int64)
        a, b = perm[rows, j].copy(), perm[rows, pick].copy()
        perm[rows, j], perm[rows, pick] = b, a
    return perm[:, :k].astype(np.int32)


def token_ids(seed: int, T: int, vocab: int) -> np.ndarray:
    """T token ids uniform over [0, vocab), int32."""
    return (splitmix64(seed, 7, T) % np.uint64(vocab)).astype(np.int32)
