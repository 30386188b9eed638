"""Float64 CPU oracle for the HARP rotate + quantize path -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
import this package. It wraps ``oracle.c`` (plain C, float64) with ctypes and
shares no code with the CUDA library. Block construction from the raw draws
(Sylvester Hadamard, QR, Cayley, Givens) lives in the C file too, so the
oracle's blocks are its own.

Parity pins: every function here is checked against closed forms, library
routines, brute force or published values in ``tests/test_oracle.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

LLOYD_MAX = 0
ABSMAX = 1
KINDS = {"lloyd_max": LLOYD_MAX, "absmax": ABSMAX}
BLOCK_KINDS = {"hadamard": 0, "qr": 1, "cayley_hadamard": 2}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, no fast-math; OpenMP
    spreads its independent rows / columns over the host threads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-fopenmp",
                               "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _set_types(_lib)
    return _lib


_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_I8 = ctypes.POINTER(ctypes.c_int8)
_U16 = ctypes.POINTER(ctypes.c_uint16)
_INT = ctypes.c_int
_L = ctypes.c_int64


def _set_types(L):
    L.orc_apply.argtypes = [_L, _INT, _I32, _D, _D, _INT, _D, _D]
    L.orc_rotate_rows.argtypes = [_L, _L, _INT, _I32, _D, _D, _INT, _D, _D]
    L.orc_rotate_cols.argtypes = [_L, _L, _INT, _I32, _D, _D, _INT, _D, _D]
    L.orc_dense.argtypes = [_L, _INT, _I32, _D, _D, _D]
    L.orc_sylvester.argtypes = [_INT, _D]
    L.orc_qr_q.argtypes = [_INT, _D, _D]
    L.orc_cayley.argtypes = [_INT, _D, _D]
    L.orc_givens.argtypes = [ctypes.c_double, _D]
    L.orc_givens.restype = None
    L.orc_stage_blocks.argtypes = [_INT, _INT, _L, _D, _D, ctypes.c_double, _D]
    L.orc_theta_quantize.argtypes = [_L, _D, _I8, ctypes.POINTER(ctypes.c_float)]
    L.orc_theta_blocks.argtypes = [_INT, _L, _I8, ctypes.c_double, _D, _D]
    L.orc_round_mid.argtypes = [_INT, _L, _D, _D]
    L.orc_lloyd_max.argtypes = [_INT, _D, ctypes.POINTER(ctypes.c_int)]
    L.orc_f16_bits.argtypes = [ctypes.c_double]
    L.orc_f16_bits.restype = ctypes.c_uint16
    L.orc_f16_value.argtypes = [ctypes.c_uint16]
    L.orc_f16_value.restype = ctypes.c_double
    L.orc_quantize.argtypes = [_INT, _INT, _L, _L, _L, _D, _U8, _U16, _D, _D]
    L.orc_quantize_mode.argtypes = [_INT, _INT, _L, _INT, _L, _L, _D, _U8, _U16, _D, _D]
    L.orc_dequantize.argtypes = [_INT, _INT, _L, _L, _L, _U8, _U16, _D]
    L.orc_pack.argtypes = [_INT, _L, _L, _U8, _U8]
    L.orc_unpack.argtypes = [_INT, _L, _L, _U8, _U8]
    L.orc_threads.argtypes = [_INT]
    L.orc_threads.restype = _INT
    L.orc_two_sided_rows.argtypes = [_L, _L, _INT, _I32, _D, _D, _INT, _I32, _D, _D, _D, _L, _I64, _D]
    L.orc_inverse_rows.argtypes = [_L, _L, _INT, _I32, _D, _D, _INT, _I32, _D, _D, _D, _L, _I64, _D]


def threads(n: int = 0) -> int:
    """Set the number of host threads of the oracle's row / column loops
    (n <= 0: unchanged); returns the current number."""
    return int(lib().orc_threads(int(n)))


def _p(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def _chk(st, what):
    if st != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


class Processor:
    """A processor (radix schedule, float64 blocks, signs) in the oracle's hands."""

    def __init__(self, radix, blocks, signs=None):
        self.radix = np.ascontiguousarray(radix, dtype=np.int32)
        self.d = int(np.prod(self.radix))
        self.blocks = np.ascontiguousarray(np.concatenate([np.asarray(b, np.float64).ravel()
                                                           for b in blocks]))
        assert self.blocks.size == self.d * int(self.radix.sum())
        self.signs = None if signs is None else np.ascontiguousarray(signs, dtype=np.float64)

    @property
    def m(self):
        return int(self.radix.size)

    def stage_blocks(self, t):
        off = self.d * int(self.radix[:t].sum())
        b = int(self.radix[t])
        return self.blocks[off: off + self.d * b].reshape(self.d // b, b, b)

    def apply(self, x, inverse=False):
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty_like(x)
        _chk(lib().orc_apply(self.d, self.m, _p(self.radix, _I32), _p(self.blocks, _D),
                             _p(self.signs, _D), int(inverse), _p(x, _D), _p(y, _D)), "apply")
        return y

    def rotate_rows(self, X, inverse=False):
        X = np.ascontiguousarray(X, dtype=np.float64)
        Y = np.empty_like(X)
        _chk(lib().orc_rotate_rows(X.shape[0], X.shape[1], self.m, _p(self.radix, _I32),
                                   _p(self.blocks, _D), _p(self.signs, _D), int(inverse),
                                   _p(X, _D), _p(Y, _D)), "rotate_rows")
        return Y

    def rotate_cols(self, X, inverse=False):
        X = np.ascontiguousarray(X, dtype=np.float64)
        Y = np.empty_like(X)
        _chk(lib().orc_rotate_cols(X.shape[0], X.shape[1], self.m, _p(self.radix, _I32),
                                   _p(self.blocks, _D), _p(self.signs, _D), int(inverse),
                                   _p(X, _D), _p(Y, _D)), "rotate_cols")
        return Y

    def dense(self):
        out = np.empty((self.d, self.d), dtype=np.float64)
        _chk(lib().orc_dense(self.d, self.m, _p(self.radix, _I32), _p(self.blocks, _D),
                             _p(self.signs, _D), _p(out, _D)), "dense")
        return out


def sylvester(b):
    out = np.empty((b, b), dtype=np.float64)
    _chk(lib().orc_sylvester(b, _p(out, _D)), "sylvester")
    return out


def qr_q(G):
    G = np.ascontiguousarray(G, dtype=np.float64)
    out = np.empty_like(G)
    _chk(lib().orc_qr_q(G.shape[0], _p(G, _D), _p(out, _D)), "qr_q")
    return out


def cayley(A):
    A = np.ascontiguousarray(A, dtype=np.float64)
    out = np.empty_like(A)
    _chk(lib().orc_cayley(A.shape[0], _p(A, _D), _p(out, _D)), "cayley")
    return out


def givens(angle):
    out = np.empty((2, 2), dtype=np.float64)
    lib().orc_givens(float(angle), _p(out, _D))
    return out


def stage_blocks(kind, b, n_groups, gauss=None, base=None, skew_scale=0.0):
    out = np.empty((n_groups, b, b), dtype=np.float64)
    g = None if gauss is None else np.ascontiguousarray(gauss, dtype=np.float64)
    bs = None if base is None else np.ascontiguousarray(base, dtype=np.float64)
    _chk(lib().orc_stage_blocks(BLOCK_KINDS[kind], b, n_groups, _p(g, _D), _p(bs, _D),
                                float(skew_scale), _p(out, _D)), "stage_blocks")
    return out


def theta_quantize(theta):
    """int8 storage of one stage's parameters: (q int8, scale float32)."""
    t = np.ascontiguousarray(theta, dtype=np.float64).ravel()
    q = np.empty(t.size, dtype=np.int8)
    s = ctypes.c_float(0.0)
    _chk(lib().orc_theta_quantize(t.size, _p(t, _D), _p(q, _I8), ctypes.byref(s)), "theta_quantize")
    return q.reshape(np.shape(theta)), np.float32(s.value)


def theta_blocks(b, q, scale, G=None):
    """Blocks [n_groups, b, b] of one stage from int8 q [n_groups, b(b-1)/2]
    (b = 2: [n_groups, 1]) and the float scale; G the base mixer or None for
    the normalised Sylvester matrix."""
    P = max(b * (b - 1) // 2, 1) if b > 1 else 0
    q = np.ascontiguousarray(q, dtype=np.int8)
    n = int(q.shape[0])
    if q.size != n * P:
        raise ValueError("oracle: theta_blocks wants [n_groups, b(b-1)/2] values")
    out = np.empty((n, b, b), dtype=np.float64)
    g = None if G is None else np.ascontiguousarray(G, dtype=np.float64)
    _chk(lib().orc_theta_blocks(b, n, _p(q, _I8), float(np.float32(scale)), _p(g, _D),
                                _p(out, _D)), "theta_blocks")
    return out


def processor(side) -> Processor:
    """The oracle's own float64 processor for a ``synth.Side`` of raw draws."""
    d = side.d
    blocks = []
    for t, b in enumerate(side.radix):
        base = side.base[t] if side.base else None
        blocks.append(stage_blocks(side.block_kind, b, d // b, side.gauss[t], base,
                                   side.skew_scale))
    return Processor(side.radix, blocks, side.signs)


def lloyd_max(bits):
    c = np.empty(1 << bits, dtype=np.float64)
    it = ctypes.c_int(0)
    _chk(lib().orc_lloyd_max(bits, _p(c, _D), ctypes.byref(it)), "lloyd_max")
    return c, it.value


def f16_bits(x):
    return int(lib().orc_f16_bits(float(x)))


def f16_value(h):
    return float(lib().orc_f16_value(int(h)))


SCALE_MODES = {"rms": 0, "absmax": 1}


def quantize(kind, bits, group, X, with_margins=True, scale_mode="rms"):
    """Group-wise codes and fp16 scales of X; scale_mode 'rms' (default) or
    'absmax' (Lloyd-Max only: s = max|x| / largest centroid)."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    rows, cols = X.shape
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty((rows, cols // group), dtype=np.uint16)
    margin = np.empty((rows, cols), dtype=np.float64) if with_margins else None
    smargin = np.empty((rows, cols // group), dtype=np.float64) if with_margins else None
    _chk(lib().orc_quantize_mode(KINDS[kind], bits, group, SCALE_MODES[scale_mode], rows, cols, _p(X, _D),
                                 _p(codes, _U8), _p(scales, _U16), _p(margin, _D), _p(smargin, _D)), "quantize")
    return codes, scales, margin, smargin


def dequantize(kind, bits, group, codes, scales):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    rows, cols = codes.shape
    X = np.empty((rows, cols), dtype=np.float64)
    _chk(lib().orc_dequantize(KINDS[kind], bits, group, rows, cols, _p(codes, _U8),
                              _p(scales, _U16), _p(X, _D)), "dequantize")
    return X


def pack(bits, codes):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    out = np.empty((rows, cols * bits // 8), dtype=np.uint8)
    _chk(lib().orc_pack(bits, rows, cols, _p(codes, _U8), _p(out, _U8)), "pack")
    return out


def unpack(bits, packed, cols):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    out = np.empty((rows, cols), dtype=np.uint8)
    _chk(lib().orc_unpack(bits, rows, cols, _p(packed, _U8), _p(out, _U8)), "unpack")
    return out


def _side_args(P):
    if P is None:
        return 0, None, None, None
    return P.m, _p(P.radix, _I32), _p(P.blocks, _D), _p(P.signs, _D)


def two_sided_rows(W, left, right, which):
    """Rows ``which`` of M_L W M_R^T (left may be None)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    which = np.ascontiguousarray(which, dtype=np.int64)
    out = np.empty((which.size, W.shape[1]), dtype=np.float64)
    _chk(lib().orc_two_sided_rows(W.shape[0], W.shape[1], *_side_args(left), *_side_args(right),
                                  _p(W, _D), which.size, _p(which, _I64), _p(out, _D)),
         "two_sided_rows")
    return out


def inverse_rows(Wp, left, right, which):
    """Rows ``which`` of M_L^T W' M_R (left may be None)."""
    Wp = np.ascontiguousarray(Wp, dtype=np.float64)
    which = np.ascontiguousarray(which, dtype=np.int64)
    out = np.empty((which.size, Wp.shape[1]), dtype=np.float64)
    _chk(lib().orc_inverse_rows(Wp.shape[0], Wp.shape[1], *_side_args(left), *_side_args(right),
                                _p(Wp, _D), which.size, _p(which, _I64), _p(out, _D)),
         "inverse_rows")
    return out


def rotate_quantize(X, left, right, kind, bits, group):
    """Full two-sided (or right-only) rotate + quantize in float64.
    Returns (rotated, codes, packed, scales, margin, scale_margin)."""
    Y = X if left is None else left.rotate_cols(X)
    Y = right.rotate_rows(Y)
    codes, scales, margin, smargin = quantize(kind, bits, group, Y)
    return Y, codes, pack(bits, codes), scales, margin, smargin


MID_KINDS = {"f32": 0, "bf16": 1, "f16": 2}


def round_mid(kind, X):
    """X rounded (nearest even) to the storage type `kind` ('f32' | 'bf16' |
    'f16', fp16 saturating at 65504), as float64."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    out = np.empty_like(X)
    _chk(lib().orc_round_mid(MID_KINDS[kind], X.size, _p(X, _D), _p(out, _D)), "round_mid")
    return out


def requantize(codes, scales, right, kind_in, bits_in, group_in, mid, kind_out, bits_out, group_out):
    """PolarQuant's two-stage codec [PQ 2-3]: dequantise the first-stage codes,
    rotate the rows back, store the restored weights as `mid`, then quantise
    them (no rotation) with the second quantiser.
    Returns (restored, codes, packed, scales, margin, scale_margin)."""
    Y = round_mid(mid, right.rotate_rows(dequantize(kind_in, bits_in, group_in, codes, scales),
                                         inverse=True))
    c2, s2, margin, smargin = quantize(kind_out, bits_out, group_out, Y)
    return Y, c2, pack(bits_out, c2), s2, margin, smargin


def dequantize_unrotate(codes, scales, left, right, kind, bits, group):
    Xq = dequantize(kind, bits, group, codes, scales)
    Y = right.rotate_rows(Xq, inverse=True)
    return Y if left is None else left.rotate_cols(Y, inverse=True)
