"""Seeded synthetic inputs for the HARP rotate+quantize workloads.

This module only draws random numbers and lays them out: data matrices with
the distributions and outlier structure of the five workloads, +-1 sign
vectors, and the raw Gaussian draws from which each side builds its own
orthogonal blocks. It holds none of the method's arithmetic (no Hadamard,
QR, Cayley, rotation or quantisation); both the CUDA library's tests and the
float64 oracle read the same bytes from here.

Generator: a counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; the finaliser constants are the
published ones). Element ``i`` of stream ``(seed, stream)`` is
``mix(key + (i + 1) * GAMMA)`` with ``key = mix(seed * GAMMA ^ stream)``, so
any element can be recomputed on its own. Uniforms are ``((u >> 11) + 0.5) *
2**-53`` in (0, 1); normals use the Box-Muller cosine branch on uniforms
``2i`` and ``2i + 1``.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# Stream identifiers: one per independent draw of a workload.
S_DATA = 1
S_DATA_AUX = 2       # second uniform stream (chi-square / Laplace sign)
S_DATA_AUX2 = 3
S_OUTLIER = 4        # permutation choosing outlier channels / rows
S_SIGNS_R = 5
S_SIGNS_L = 6
S_BLOCKS_R = 100     # + stage index: per-group Gaussian draws, right side
S_BLOCKS_L = 200     # + stage index: per-group Gaussian draws, left side
S_BASE_R = 300       # + stage index: one fixed Gaussian per stage (QR base mixer)
S_BASE_L = 400

CHUNK = 1 << 22


def _mix_scalar(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return _mix_scalar(((seed * 0x9E3779B97F4A7C15) & _MASK64) ^ stream)


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def raw_u64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """Elements [offset, offset + n) of the raw 64-bit stream."""
    key = np.uint64(stream_key(seed, stream))
    out = np.empty(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for a in range(0, n, CHUNK):
            b = min(n, a + CHUNK)
            i = np.arange(offset + a + 1, offset + b + 1, dtype=np.uint64)
            out[a:b] = _mix(key + i * GAMMA)
    return out


def uniform(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    u = raw_u64(seed, stream, n, offset)
    return ((u >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    for a in range(0, n, CHUNK):
        b = min(n, a + CHUNK)
        u = uniform(seed, stream, 2 * (b - a), 2 * (offset + a))
        out[a:b] = np.sqrt(-2.0 * np.log(u[0::2])) * np.cos(2.0 * math.pi * u[1::2])
    return out


def student_t(seed: int, nu: int, n: int, offset: int = 0) -> np.ndarray:
    """t_nu = Z / sqrt(chi2_nu / nu); chi2 of even order from -2 ln of uniforms,
    odd order adds one squared normal."""
    z = normal(seed, S_DATA, n, offset)
    chi = np.zeros(n, dtype=np.float64)
    for p in range(nu // 2):
        chi += -2.0 * np.log(uniform(seed, S_DATA_AUX + 16 * p, n, offset))
    if nu % 2:
        chi += normal(seed, S_DATA_AUX2, n, offset) ** 2
    return z / np.sqrt(chi / nu)


def laplace(seed: int, scale: float, n: int, offset: int = 0) -> np.ndarray:
    """Laplace(0, scale) with scale the b parameter (std = scale * sqrt 2)."""
    u = uniform(seed, S_DATA, n, offset)
    return np.where(u < 0.5, scale * np.log(2.0 * u), -scale * np.log(2.0 * (1.0 - u)))


def choose(seed: int, stream: int, n: int, k: int) -> np.ndarray:
    """k distinct indices of [0, n), a seeded permutation's first k entries."""
    return np.sort(np.argsort(raw_u64(seed, stream, n), kind="stable")[:k])


def signs(seed: int, stream: int, d: int) -> np.ndarray:
    """+-1.0 per coordinate from the top bit of the raw stream."""
    u = raw_u64(seed, stream, d)
    return np.where((u >> np.uint64(63)) == 0, 1.0, -1.0).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (round to nearest even) -> bfloat16 bits (RNE)."""
    f = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (f + np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- workloads

@dataclasses.dataclass
class Side:
    """Raw draws for one processor: radix schedule, signs and per-stage
    Gaussians. ``block_kind`` says how each side turns draws into blocks:
    'hadamard' (the base mixer G_b in every group), 'qr' (Q of the QR of each
    group's Gaussian) or 'cayley_hadamard' (Cayley map of the skew matrix from
    each group's Gaussian, scaled by ``skew_scale``, times G_b). G_b is the
    normalised Sylvester Hadamard for b a power of two, else the Q factor of
    the stage's fixed Gaussian in ``base``.
    """

    radix: tuple
    signs: np.ndarray            # float32 [d]
    block_kind: str
    gauss: list                  # per stage: float64 [d / b_t, b_t, b_t] or None
    skew_scale: float = 0.0
    base: list = None            # per stage: float64 [b_t, b_t] fixed Gaussian for
                                 # the base mixer of a non-power-of-two radix, or None

    @property
    def d(self) -> int:
        return int(np.prod(self.radix))


@dataclasses.dataclass
class Quant:
    kind: str        # 'lloyd_max' | 'absmax'
    bits: int
    group: int


@dataclasses.dataclass
class Workload:
    name: str
    rows: int
    cols: int
    dtype: str               # 'f32' | 'bf16'
    x: np.ndarray            # float32 [rows, cols] or uint16 bf16 bits
    right: Side
    left: Side | None
    quants: list


def side_draws(seed: int, radix, block_kind: str, sign_stream: int,
               block_stream: int, skew_scale: float = 0.0,
               sign_seed: int | None = None) -> Side:
    d = int(np.prod(radix))
    sg = signs(seed if sign_seed is None else sign_seed, sign_stream, d)
    gauss, base = [], []
    for t, b in enumerate(radix):
        if block_kind == "hadamard":
            gauss.append(None)
        else:
            g = normal(seed, block_stream + t, (d // b) * b * b)
            gauss.append(g.reshape(d // b, b, b))
        if block_kind != "qr" and (b & (b - 1)) != 0:
            base.append(normal(seed, block_stream + 200 + t, b * b).reshape(b, b))
        else:
            base.append(None)
    return Side(tuple(radix), sg, block_kind, gauss, skew_scale, base)


def x_as_f64(w: Workload) -> np.ndarray:
    if w.dtype == "bf16":
        return bf16_bits_to_f64(w.x)
    return w.x.astype(np.float64)


def workload(name: str, tokens: int = 8192) -> Workload:
    """The five synthetic workloads by name: 'c1' .. 'c5'. Seeds are fixed."""
    if name == "c1":
        # 64x256 fp32 N(0,1), 2 columns x20; (16,16) Sylvester blocks; signs
        # from seed 0; 3-bit Lloyd-Max, group 128, RMS scale.
        rows, cols, seed = 64, 256, 1
        x = normal(seed, S_DATA, rows * cols).reshape(rows, cols)
        x[:, choose(seed, S_OUTLIER, cols, 2)] *= 20.0
        right = side_draws(seed, (16, 16), "hadamard", S_SIGNS_R, S_BLOCKS_R, sign_seed=0)
        return Workload(name, rows, cols, "f32", x.astype(np.float32), right, None,
                        [Quant("lloyd_max", 3, 128)])
    if name == "c2":
        rows = cols = 4096
        seed = 2
        x = (0.02 * student_t(seed, 3, rows * cols)).reshape(rows, cols)
        x[:, choose(seed, S_OUTLIER, cols, round(0.005 * cols))] *= 20.0
        right = side_draws(seed, (16, 16, 16), "qr", S_SIGNS_R, S_BLOCKS_R)
        left = side_draws(seed, (16, 16, 16), "qr", S_SIGNS_L, S_BLOCKS_L)
        return Workload(name, rows, cols, "bf16", to_bf16_bits(x), right, left,
                        [Quant("lloyd_max", 2, 128), Quant("lloyd_max", 4, 128)])
    if name == "c3":
        rows, cols, seed = tokens, 4096, 3
        x = normal(seed, S_DATA, rows * cols).reshape(rows, cols)
        x[:, choose(seed, S_OUTLIER, cols, 4)] *= 50.0
        right = side_draws(seed, (8, 8, 8, 8), "cayley_hadamard", S_SIGNS_R, S_BLOCKS_R,
                           skew_scale=0.05)
        return Workload(name + f"_T{tokens}", rows, cols, "bf16", to_bf16_bits(x), right, None,
                        [Quant("absmax", 4, cols)])
    if name == "c4":
        rows, cols, seed = 4096, 11008, 4
        x = laplace(seed, 0.02, rows * cols).reshape(rows, cols)
        right = side_draws(seed, (43, 16, 16), "qr", S_SIGNS_R, S_BLOCKS_R)
        left = side_draws(seed, (16, 16, 16), "qr", S_SIGNS_L, S_BLOCKS_L)
        return Workload(name, rows, cols, "bf16", to_bf16_bits(x), right, left,
                        [Quant("lloyd_max", 3, 128)])
    if name == "c5":
        rows, cols, seed = 8192, 28672, 5
        x = (0.015 * student_t(seed, 4, rows * cols)).reshape(rows, cols)
        x[choose(seed, S_OUTLIER, rows, round(0.01 * rows)), :] *= 10.0
        right = side_draws(seed, (7, 16, 16, 16), "qr", S_SIGNS_R, S_BLOCKS_R)
        left = side_draws(seed, (32, 16, 16), "qr", S_SIGNS_L, S_BLOCKS_L)
        return Workload(name, rows, cols, "bf16", to_bf16_bits(x), right, left,
                        [Quant("lloyd_max", 2, 64), Quant("absmax", 4, 128)])
    raise KeyError(name)


def small_matrix(seed: int, rows: int, cols: int, outlier_cols: int = 0,
                 scale: float = 1.0) -> np.ndarray:
    """A small N(0, scale^2) float64 matrix with a few columns x20 (test cases)."""
    x = scale * normal(seed, S_DATA, rows * cols).reshape(rows, cols)
    if outlier_cols:
        x[:, choose(seed, S_OUTLIER, cols, outlier_cols)] *= 20.0
    return x


S_THETA = 500       # + stage index: int8-stored stage parameters


def theta_draws(seed: int, stage: int, n_groups: int, b: int, spread: float = 40.0):
    """Stored int8 stage parameters: [n_groups, b(b-1)/2] values (one for
    b = 2, none for b = 1), rint(spread * N(0,1)) clipped to [-127, 127], as a
    trained stage kept in int8 would look."""
    p = b * (b - 1) // 2 if b > 2 else (1 if b == 2 else 0)
    g = normal(seed, S_THETA + stage, n_groups * p)
    return np.clip(np.rint(spread * g), -127, 127).astype(np.int8).reshape(n_groups, p)


def random_code_stream(seed: int, rows: int, cols: int, bits: int, group: int,
                       scale_lo: float = 0.01, scale_hi: float = 0.05):
    """Random inputs for the inverse path: packed code bytes (any byte string
    is a valid LSB-first code stream, so uniform bytes are uniform codes) and
    fp16 scale bits uniform in [scale_lo, scale_hi)."""
    nbytes = cols * bits // 8
    raw = raw_u64(seed, 1, rows * nbytes).astype(np.uint8).reshape(rows, nbytes)
    u = uniform(seed, 2, rows * (cols // group)).reshape(rows, cols // group)
    sc = (scale_lo + (scale_hi - scale_lo) * u).astype(np.float16).view(np.uint16)
    return raw, sc
