"""Python binding of libharp (HARP rotate + quantize on B200, sm_100a).

Argument marshalling only: every step of the path runs in the CUDA library
(``libharp.so``, declared in ``include/harp.h``); PyTorch supplies device
memory and streams. Importing this package does not need a GPU; calling a
compute function without the built library or without a CUDA device raises.

The C entry points keep their names here (``harp_rotate``,
``harp_rotate_quantize``, ...). ``Plan`` and ``Codebook`` own the C objects.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libharp.so")

HARP_OK = 0
HARP_F32, HARP_BF16, HARP_F16 = 0, 1, 2
HARP_RIGHT, HARP_LEFT = 0, 1
HARP_FWD, HARP_INV = 0, 1
HARP_LLOYD_MAX, HARP_ABSMAX = 0, 1
HARP_BLOCKS_HADAMARD, HARP_BLOCKS_QR, HARP_BLOCKS_CAYLEY = 0, 1, 2
HARP_MAX_STAGES = 16
HARP_STATIC_WORKSPACE_BYTES = 32 << 20

BLOCK_KINDS = {"hadamard": HARP_BLOCKS_HADAMARD, "qr": HARP_BLOCKS_QR,
               "cayley_hadamard": HARP_BLOCKS_CAYLEY}
QUANT_KINDS = {"lloyd_max": HARP_LLOYD_MAX, "absmax": HARP_ABSMAX}

# every symbol include/harp.h declares
EXPORTS = (
    "harp_status_string", "harp_version", "harp_plan_create", "harp_plan_destroy",
    "harp_plan_info", "harp_stage_blocks", "harp_lloyd_max_centroids",
    "harp_codebook_create", "harp_codebook_destroy", "harp_codebook_tables",
    "harp_workspace_size", "harp_rotate", "harp_quantize", "harp_dequantize",
    "harp_rotate_quantize", "harp_dequantize_unrotate", "harp_rotate_quantize_static",
    "harp_pass_count", "harp_pass_fma", "harp_set_pass_events",
    "harp_theta_blocks", "harp_plan_load_theta", "harp_requantize", "harp_fault_status",
    "harp_set_block_stages", "harp_host_scratch_size", "harp_rotate_quantize_host",
    "harp_dequantize_unrotate_host",
)


class HarpError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def lib():
    """Load libharp.so (built by ``build.build()``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libharp.so not built at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        L.harp_status_string.restype = ctypes.c_char_p
        L.harp_status_string.argtypes = [_INT]
        L.harp_plan_create.argtypes = [ctypes.POINTER(_P), _I64, _INT, ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.POINTER(ctypes.c_float)),
                                       ctypes.POINTER(ctypes.c_float), _P]
        L.harp_plan_destroy.argtypes = [_P]
        L.harp_plan_info.argtypes = [_P, ctypes.POINTER(_I64), ctypes.POINTER(_INT),
                                     ctypes.POINTER(ctypes.c_int32)]
        L.harp_stage_blocks.argtypes = [_INT, _INT, _I64, _P, _P, ctypes.c_double, _P]
        L.harp_lloyd_max_centroids.argtypes = [_INT, _P]
        L.harp_codebook_create.argtypes = [ctypes.POINTER(_P), _INT, _INT, _I64, _INT, _P]
        L.harp_codebook_destroy.argtypes = [_P]
        L.harp_codebook_tables.argtypes = [_P, _P, _P]
        L.harp_workspace_size.argtypes = [_P, _P, _I64, _I64, ctypes.POINTER(ctypes.c_size_t)]
        L.harp_rotate.argtypes = [_P, _INT, _INT, _P, _INT, _P, _INT, _I64, _I64, _I64, _I64, _P]
        L.harp_quantize.argtypes = [_P, _P, _INT, _I64, _I64, _I64, _P, _P, _P]
        L.harp_dequantize.argtypes = [_P, _P, _P, _I64, _I64, _P, _INT, _I64, _P]
        L.harp_rotate_quantize.argtypes = [_P, _P, _P, _P, _INT, _I64, _I64, _P, _P, _P, _P,
                                           ctypes.c_size_t, _P]
        L.harp_dequantize_unrotate.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _P, _INT, _P,
                                               ctypes.c_size_t, _P]
        L.harp_pass_count.argtypes = [_P, _P, _P, ctypes.POINTER(_INT)]
        L.harp_pass_fma.argtypes = [_P, _P, _P, _INT, ctypes.POINTER(_INT)]
        L.harp_set_pass_events.argtypes = [_P, _INT]
        L.harp_rotate_quantize_static.argtypes = [_P, _P, _P, _P, _INT, _I64, _I64, _P, _P, _P, _P]
        L.harp_theta_blocks.argtypes = [_INT, _I64, _P, ctypes.c_float, _P, _P, _P]
        L.harp_plan_load_theta.argtypes = [_P, _INT, _P, ctypes.c_float, _P, _P]
        L.harp_requantize.argtypes = [_P, _P, _P, _P, _I64, _I64, _INT, _P, _P, _P, _P, _P]
        L.harp_fault_status.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        L.harp_set_block_stages.argtypes = [_INT]
        L.harp_host_scratch_size.argtypes = [_P, _P, _P, _I64, _I64, _INT, ctypes.POINTER(ctypes.c_size_t)]
        L.harp_rotate_quantize_host.argtypes = [_P, _P, _P, _P, _INT, _I64, _I64, _P, _P, _P, ctypes.c_size_t, _P]
        L.harp_dequantize_unrotate_host.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _P, _INT, _P,
                                                    ctypes.c_size_t, _P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().harp_status_string(int(status)).decode()


def _check(status, what):
    if status != HARP_OK:
        raise HarpError(status, what)


# ------------------------------------------------------------ host helpers

def stage_blocks(kind, b, n_groups, gauss=None, base=None, skew_scale=0.0) -> np.ndarray:
    """float32 [n_groups, b, b] blocks of one stage from raw Gaussian draws."""
    out = np.empty((n_groups, b, b), dtype=np.float32)
    g = None if gauss is None else np.ascontiguousarray(gauss, dtype=np.float64)
    bs = None if base is None else np.ascontiguousarray(base, dtype=np.float64)
    kind = BLOCK_KINDS.get(kind, kind)
    _check(lib().harp_stage_blocks(kind, b, n_groups, None if g is None else g.ctypes.data,
                                   None if bs is None else bs.ctypes.data, float(skew_scale),
                                   out.ctypes.data), "harp_stage_blocks")
    return out


def lloyd_max_centroids(bits: int) -> np.ndarray:
    out = np.empty(1 << bits, dtype=np.float32)
    _check(lib().harp_lloyd_max_centroids(bits, out.ctypes.data), "harp_lloyd_max_centroids")
    return out


class Plan:
    """A processor plan (radix schedule, float32 blocks, signs) on the current device."""

    def __init__(self, radix, blocks, signs=None, stream=None):
        radix = [int(b) for b in radix]
        self.radix = tuple(radix)
        self.d = int(np.prod(radix))
        self._blocks = [np.ascontiguousarray(b, dtype=np.float32) for b in blocks]
        self._signs = None if signs is None else np.ascontiguousarray(signs, dtype=np.float32)
        rad = (ctypes.c_int32 * len(radix))(*radix)
        ptrs = (ctypes.POINTER(ctypes.c_float) * len(radix))(
            *[b.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) for b in self._blocks])
        h = _P()
        _check(lib().harp_plan_create(ctypes.byref(h), self.d, len(radix), rad, ptrs,
                                      None if self._signs is None else
                                      self._signs.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                      _stream(stream)),
               "harp_plan_create")
        self.handle = h

    @classmethod
    def from_side(cls, side) -> "Plan":
        """Build the library's own blocks from a ``synth.Side`` of raw draws."""
        blocks = []
        for t, b in enumerate(side.radix):
            base = side.base[t] if side.base else None
            blocks.append(stage_blocks(side.block_kind, b, side.d // b, side.gauss[t], base,
                                       side.skew_scale))
        return cls(side.radix, blocks, side.signs)

    def info(self):
        d, m = _I64(), _INT()
        rad = (ctypes.c_int32 * HARP_MAX_STAGES)()
        _check(lib().harp_plan_info(self.handle, ctypes.byref(d), ctypes.byref(m), rad), "harp_plan_info")
        return d.value, m.value, tuple(rad[: m.value])

    def close(self):
        if getattr(self, "handle", None) and self.handle.value:
            lib().harp_plan_destroy(self.handle)
            self.handle = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


SCALE_MODES = {"rms": 0, "absmax": 1}


class Codebook:
    """Quantizer description: kind ('lloyd_max' | 'absmax'), bits, group,
    Lloyd-Max scale mode ('rms' default | 'absmax')."""

    def __init__(self, kind, bits, group, centroids=None, scale_mode="rms"):
        self.kind = QUANT_KINDS.get(kind, kind)
        self.bits, self.group = int(bits), int(group)
        self.scale_mode = SCALE_MODES.get(scale_mode, scale_mode)
        c = None if centroids is None else np.ascontiguousarray(centroids, dtype=np.float32)
        h = _P()
        _check(lib().harp_codebook_create(ctypes.byref(h), self.kind, self.bits, self.group, self.scale_mode,
                                          None if c is None else c.ctypes.data), "harp_codebook_create")
        self.handle = h

    def tables(self):
        K = 1 << self.bits
        c = np.empty(K, dtype=np.float32)
        t = np.zeros(K - 1, dtype=np.float32)
        _check(lib().harp_codebook_tables(self.handle, c.ctypes.data, t.ctypes.data), "harp_codebook_tables")
        return c, t

    def close(self):
        if getattr(self, "handle", None) and self.handle.value:
            lib().harp_codebook_destroy(self.handle)
            self.handle = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def workspace_size(left, right, rows, cols) -> int:
    n = ctypes.c_size_t()
    _check(lib().harp_workspace_size(left.handle if left else None, right.handle if right else None,
                                     rows, cols, ctypes.byref(n)), "harp_workspace_size")
    return n.value


# ------------------------------------------------------------ device calls

def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return HARP_F32
    if t.dtype == torch.bfloat16:
        return HARP_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    import torch
    if stream is None:
        if not torch.cuda.is_available():
            return None            # the library reports the missing device itself
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libharp compute calls take CUDA tensors")


def harp_rotate(plan, side, direction, x, out, stream=None):
    """out = x with the processor applied to rows (HARP_RIGHT) or columns
    (HARP_LEFT); direction HARP_FWD (M) or HARP_INV (M^T). 2-D tensors."""
    _require_cuda(x, out)
    rows, cols = x.shape
    _check(lib().harp_rotate(plan.handle, side, direction, _ptr(x), _dtype_code(x), _ptr(out),
                             _dtype_code(out), rows, cols, x.stride(0), out.stride(0), _stream(stream)),
           "harp_rotate")
    return out


def harp_quantize(cb, x, codes, scales, stream=None):
    _require_cuda(x, codes, scales)
    rows, cols = x.shape
    _check(lib().harp_quantize(cb.handle, _ptr(x), _dtype_code(x), rows, cols, x.stride(0),
                               _ptr(codes), _ptr(scales), _stream(stream)), "harp_quantize")
    return codes, scales


def harp_dequantize(cb, codes, scales, out, stream=None):
    _require_cuda(codes, scales, out)
    rows, cols = out.shape
    _check(lib().harp_dequantize(cb.handle, _ptr(codes), _ptr(scales), rows, cols, _ptr(out),
                                 _dtype_code(out), out.stride(0), _stream(stream)), "harp_dequantize")
    return out


def harp_rotate_quantize(left, right, cb, x, codes, scales, rotated_out=None, workspace=None,
                         stream=None):
    _require_cuda(x, codes, scales, rotated_out, workspace)
    rows, cols = x.shape
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().harp_rotate_quantize(left.handle if left else None, right.handle, cb.handle,
                                      _ptr(x), _dtype_code(x), rows, cols, _ptr(codes), _ptr(scales),
                                      _ptr(rotated_out), _ptr(workspace), ws, _stream(stream)),
           "harp_rotate_quantize")
    return codes, scales


def harp_pass_count(left, right, cb) -> int:
    n = ctypes.c_int()
    _check(lib().harp_pass_count(left.handle if left else None, right.handle, cb.handle, ctypes.byref(n)),
           "harp_pass_count")
    return n.value


def harp_pass_fma(left, right, cb, k) -> int:
    n = ctypes.c_int()
    _check(lib().harp_pass_fma(left.handle, right.handle, cb.handle, k, ctypes.byref(n)), "harp_pass_fma")
    return n.value


HARP_BLOCK_STAGES_AUTO, HARP_BLOCK_STAGES_TC, HARP_BLOCK_STAGES_FFMA = 0, 1, 2


def harp_set_block_stages(mode: int) -> None:
    """Block-stage arithmetic of the two-sided calls: HARP_BLOCK_STAGES_AUTO
    (per pass, the faster of the two), _TC (tensor cores, 3xTF32) or _FFMA."""
    _check(lib().harp_set_block_stages(int(mode)), "harp_set_block_stages")


def harp_fault_status() -> int:
    """The current device's record of bounded kernel waits that ran out
    (0 = none), cleared by the read. Synchronises the device."""
    v = ctypes.c_uint(0)
    _check(lib().harp_fault_status(ctypes.byref(v)), "harp_fault_status")
    return int(v.value)


_event_array = None


def harp_set_pass_events(events):
    """Time the passes of the following two-sided calls of this thread with
    torch.cuda.Event objects (enable_timing=True); [] unregisters."""
    global _event_array
    handles = []
    for e in events:
        if e.cuda_event == 0:          # torch creates the CUDA event on first record
            e.record()
        handles.append(e.cuda_event)
    _event_array = (ctypes.c_void_p * max(len(handles), 1))(*handles)
    _check(lib().harp_set_pass_events(_event_array if handles else None, len(handles)),
           "harp_set_pass_events")


def harp_rotate_quantize_static(left, right, cb, x, codes, scales, rotated_out=None, stream=None):
    """harp_rotate_quantize with the two-sided intermediate in the library's
    own device array (HARP_STATIC_WORKSPACE_BYTES): for callers that cannot
    allocate device memory. Calls on one device share that array; do not
    overlap them on the GPU."""
    _require_cuda(x, codes, scales, rotated_out)
    rows, cols = x.shape
    _check(lib().harp_rotate_quantize_static(left.handle if left else None, right.handle, cb.handle,
                                             _ptr(x), _dtype_code(x), rows, cols, _ptr(codes),
                                             _ptr(scales), _ptr(rotated_out), _stream(stream)),
           "harp_rotate_quantize_static")
    return codes, scales


def _check_theta(b, theta, n_groups, base):
    import torch
    p = b * (b - 1) // 2 if b > 2 else (1 if b == 2 else 0)
    if theta is not None and (theta.dtype != torch.int8 or not theta.is_contiguous()
                              or theta.numel() != n_groups * p):
        raise ValueError(f"theta must be a contiguous int8 tensor of {n_groups} x {p} values")
    if base is not None and (base.dtype != torch.float32 or not base.is_contiguous()
                             or base.numel() != b * b):
        raise ValueError("base must be a contiguous float32 [b, b] tensor")


def harp_theta_blocks(b, theta, theta_scale, out, base=None, stream=None):
    """Blocks [n_groups, b, b] (float32 device tensor `out`) of one stage from
    int8-stored parameters `theta` [n_groups, b(b-1)/2] (device int8) and the
    stage's float scale; `base` the float32 [b, b] base mixer on the device,
    or None for the normalised Sylvester matrix."""
    import torch
    _require_cuda(theta, out, base)
    _check_theta(b, theta, out.shape[0], base)
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape[1:]) != (b, b):
        raise ValueError("out must be a contiguous float32 [n_groups, b, b] tensor")
    n = out.shape[0]
    _check(lib().harp_theta_blocks(int(b), n, _ptr(theta), float(theta_scale), _ptr(base),
                                   _ptr(out), _stream(stream)), "harp_theta_blocks")
    return out


def harp_plan_load_theta(plan, stage, theta, theta_scale, base=None, stream=None):
    """Replace stage `stage` of `plan` with blocks built on the device from
    int8-stored parameters (see harp_theta_blocks)."""
    _require_cuda(theta, base)
    b = plan.radix[stage] if 0 <= stage < len(plan.radix) else 0
    if b:
        _check_theta(b, theta, plan.d // b, base)
    _check(lib().harp_plan_load_theta(plan.handle, int(stage), _ptr(theta), float(theta_scale),
                                      _ptr(base), _stream(stream)), "harp_plan_load_theta")
    return plan


_MID_CODES = {"f32": 0, "bf16": 1, "f16": 2}


def harp_requantize(right, cb_in, codes_in, scales_in, rows, cols, mid, cb_out, codes_out,
                    scales_out, restored_out=None, stream=None):
    """PolarQuant's two-stage codec in one pass: dequantise `codes_in` with
    cb_in, rotate the rows back with `right`, round to `mid` ('f32' | 'bf16'
    | 'f16'; optionally stored in `restored_out`), quantise with cb_out."""
    _require_cuda(codes_in, scales_in, codes_out, scales_out, restored_out)
    _check(lib().harp_requantize(right.handle, cb_in.handle, _ptr(codes_in), _ptr(scales_in), rows, cols,
                                 _MID_CODES[mid], _ptr(restored_out), cb_out.handle, _ptr(codes_out),
                                 _ptr(scales_out), _stream(stream)), "harp_requantize")
    return codes_out, scales_out


def harp_dequantize_unrotate(left, right, cb, codes, scales, out, workspace=None, stream=None):
    _require_cuda(codes, scales, out, workspace)
    rows, cols = out.shape
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().harp_dequantize_unrotate(left.handle if left else None, right.handle, cb.handle,
                                          _ptr(codes), _ptr(scales), rows, cols, _ptr(out),
                                          _dtype_code(out), _ptr(workspace), ws, _stream(stream)),
           "harp_dequantize_unrotate")
    return out


# ------------------------------------------------------------ allocating wrappers

def _require_host(*ts):
    for t in ts:
        if t is not None and t.is_cuda:
            raise ValueError("the _host calls take CPU (preferably pinned) tensors for their host buffers")


def harp_host_scratch_size(left, right, cb, rows, cols, value_dtype) -> int:
    """Device scratch bytes of harp_rotate_quantize_host /
    harp_dequantize_unrotate_host for these shapes and value dtype."""
    n = ctypes.c_size_t()
    _check(lib().harp_host_scratch_size(left.handle if left else None, right.handle, cb.handle, rows, cols,
                                        int(value_dtype), ctypes.byref(n)), "harp_host_scratch_size")
    return n.value


def empty_host_scratch(left, right, cb, rows, cols, value_dtype, device="cuda"):
    import torch
    n = harp_host_scratch_size(left, right, cb, rows, cols, value_dtype)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def harp_rotate_quantize_host(left, right, cb, x, codes, scales, scratch, stream=None):
    """harp_rotate_quantize on host buffers: x, codes and scales are CPU
    tensors (pinned for asynchronous copies), scratch a CUDA byte tensor of
    harp_host_scratch_size bytes. Enqueued on the stream; synchronise it
    before reading codes and scales."""
    _require_host(x, codes, scales)
    _require_cuda(scratch)
    rows, cols = x.shape
    _check(lib().harp_rotate_quantize_host(left.handle if left else None, right.handle, cb.handle, _ptr(x),
                                           _dtype_code(x), rows, cols, _ptr(codes), _ptr(scales), _ptr(scratch),
                                           scratch.numel() * scratch.element_size(), _stream(stream)),
           "harp_rotate_quantize_host")
    return codes, scales


def harp_dequantize_unrotate_host(left, right, cb, codes, scales, out, scratch, stream=None):
    """harp_dequantize_unrotate on host buffers (codes, scales, out CPU
    tensors; out bf16 or fp32 [rows, cols]); enqueued on the stream."""
    _require_host(codes, scales, out)
    _require_cuda(scratch)
    rows, cols = out.shape
    _check(lib().harp_dequantize_unrotate_host(left.handle if left else None, right.handle, cb.handle,
                                               _ptr(codes), _ptr(scales), rows, cols, _ptr(out), _dtype_code(out),
                                               _ptr(scratch), scratch.numel() * scratch.element_size(),
                                               _stream(stream)),
           "harp_dequantize_unrotate_host")
    return out


def empty_codes(rows, cols, cb, device="cuda"):
    import torch
    codes = torch.empty((rows, cols * cb.bits // 8), dtype=torch.uint8, device=device)
    scales = torch.empty((rows, cols // cb.group), dtype=torch.int16, device=device)
    return codes, scales


def empty_workspace(left, right, rows, cols, device="cuda"):
    import torch
    n = workspace_size(left, right, rows, cols)
    return torch.empty((max(n, 4) + 3) // 4, dtype=torch.float32, device=device)


def rotate_quantize(left, right, cb, x, want_rotated=False, stream=None):
    """Allocate outputs and run the fused forward path; returns
    (codes uint8 [rows, cols*bits/8], scales int16 fp16-bits [rows, cols/group],
    rotated fp32 or None)."""
    import torch
    rows, cols = x.shape
    codes, scales = empty_codes(rows, cols, cb, x.device)
    ws = empty_workspace(left, right, rows, cols, x.device) if left else None
    rot = torch.empty((rows, cols), dtype=torch.float32, device=x.device) if want_rotated else None
    harp_rotate_quantize(left, right, cb, x, codes, scales, rot, ws, stream)
    return codes, scales, rot


def dequantize_unrotate(left, right, cb, codes, scales, rows, cols, out_dtype=None, stream=None):
    import torch
    out = torch.empty((rows, cols), dtype=out_dtype or torch.float32, device=codes.device)
    ws = empty_workspace(left, right, rows, cols, codes.device) if left else None
    return harp_dequantize_unrotate(left, right, cb, codes, scales, out, ws, stream)
