"""Comparison helpers for the GPU-vs-oracle parity tests.

Acceptance (float32 accumulate against the float64 oracle):
  * rotated values: relative L2 error <= 2e-6 (fp32 output), 1e-2 (bf16);
  * codes: bit-exact, except elements whose oracle value x/s lies within
    1e-5 of a decision boundary (counted and reported), and groups whose
    oracle scale lies within a relative 1e-5 of an fp16 rounding boundary;
  * fp16 scales: bit-exact outside those groups;
  * packed bytes: identical wherever no excluded element touches the byte.
GPU output is decoded here with numpy bit operations, never by the oracle.
"""

from __future__ import annotations

import numpy as np

TOL_F32 = 2e-6
TOL_BF16 = 1e-2
BOUNDARY = 1e-5


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def np_unpack(packed: np.ndarray, bits: int, cols: int) -> np.ndarray:
    """LSB-first bitstream rows -> codes (uint8)."""
    rows = packed.shape[0]
    b = np.unpackbits(np.ascontiguousarray(packed, dtype=np.uint8), axis=1, bitorder="little")
    b = b[:, : cols * bits].reshape(rows, cols, bits).astype(np.uint8)
    w = (1 << np.arange(bits, dtype=np.uint8))
    return (b * w).sum(axis=2).astype(np.uint8)


def np_pack(codes: np.ndarray, bits: int) -> np.ndarray:
    rows, cols = codes.shape
    b = ((codes[..., None].astype(np.uint8) >> np.arange(bits, dtype=np.uint8)) & 1).reshape(rows, cols * bits)
    return np.packbits(b, axis=1, bitorder="little")


def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits).astype(np.uint16).view(np.float16).astype(np.float64)


def compare_quant(gpu_codes_packed, gpu_scales_bits, orc_codes, orc_scales, margin, smargin,
                  bits, group, tol=BOUNDARY):
    """Returns a report dict; raises AssertionError on a parity failure."""
    rows, cols = orc_codes.shape
    gs = np.asarray(gpu_scales_bits).astype(np.uint16).reshape(orc_scales.shape)
    gcodes = np_unpack(np.asarray(gpu_codes_packed), bits, cols)
    near_scale = smargin < tol
    scale_mismatch = (gs != orc_scales)
    bad_scale = scale_mismatch & ~near_scale
    excluded_groups = near_scale | scale_mismatch
    excl = np.repeat(excluded_groups, group, axis=1) | (margin < tol)
    code_mismatch = (gcodes != orc_codes)
    bad_codes = code_mismatch & ~excl
    merged = np.where(excl, gcodes, orc_codes)
    ref_bytes = np_pack(orc_codes, bits)
    gpu_bytes = np.asarray(gpu_codes_packed)
    touched = np.zeros(ref_bytes.shape, dtype=bool)
    er, ec = np.nonzero(excl)
    for q in range(bits):
        touched[er, (ec * bits + q) // 8] = True
    byte_bad = (gpu_bytes != ref_bytes) & ~touched
    rep = {
        "elements": int(rows * cols),
        "near_boundary": int(np.count_nonzero(margin < tol)),
        "near_scale_groups": int(np.count_nonzero(near_scale)),
        "scale_mismatch_groups": int(np.count_nonzero(scale_mismatch)),
        "code_mismatch_total": int(np.count_nonzero(code_mismatch)),
        "code_mismatch_excluded": int(np.count_nonzero(code_mismatch & excl)),
        "bad_codes": int(np.count_nonzero(bad_codes)),
        "bad_scales": int(np.count_nonzero(bad_scale)),
        "bad_bytes": int(np.count_nonzero(byte_bad)),
    }
    assert rep["bad_scales"] == 0, rep
    assert rep["bad_codes"] == 0, rep
    assert rep["bad_bytes"] == 0, rep
    # the packing of the GPU's codes is exactly its bytes (no stray bits)
    assert np.array_equal(np_pack(merged, bits), gpu_bytes), rep
    return rep
