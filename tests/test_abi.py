"""Host-side checks of the C ABI (no GPU needed): the library loads and exports
every symbol include/harp.h declares; argument checks return the documented
status before any launch; the host-built blocks and Lloyd-Max table of the
library agree with the oracle's independently built ones."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import rotation_preconditioned_bit_b200 as harp
from rotation_preconditioned_bit_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "harp.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(harp_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = harp.lib()
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(harp.EXPORTS)


def test_status_strings():
    assert harp.status_string(0) == "ok"
    for s in range(1, 8):
        assert harp.status_string(s) not in ("ok", "unknown status")
    assert harp.status_string(99) == "unknown status"
    assert harp.lib().harp_version() == 100


def test_plan_create_argument_checks():
    L = harp.lib()
    h = ctypes.c_void_p()
    rad = (ctypes.c_int32 * 2)(16, 16)
    blk = np.zeros((16, 16, 16), np.float32)
    ptrs = (ctypes.POINTER(ctypes.c_float) * 2)(*(blk.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),) * 2)
    # product of radices != d
    assert L.harp_plan_create(ctypes.byref(h), 255, 2, rad, ptrs, None, None) == 2
    # radix out of range
    rad_bad = (ctypes.c_int32 * 2)(65, 4)
    assert L.harp_plan_create(ctypes.byref(h), 260, 2, rad_bad, ptrs, None, None) == 3
    # too many stages
    assert L.harp_plan_create(ctypes.byref(h), 256, 17, rad, ptrs, None, None) == 3
    # NULL pointers
    assert L.harp_plan_create(None, 256, 2, rad, ptrs, None, None) == 1
    assert L.harp_plan_create(ctypes.byref(h), 256, 2, None, ptrs, None, None) == 1
    nullp = (ctypes.POINTER(ctypes.c_float) * 2)()
    assert L.harp_plan_create(ctypes.byref(h), 256, 2, rad, nullp, None, None) == 1
    # a vector too long for one CTA's shared memory
    rad_big = (ctypes.c_int32 * 2)(64, 1024)
    assert L.harp_plan_create(ctypes.byref(h), 65536, 2, rad_big, ptrs, None, None) in (3, 2)


def test_plan_create_without_device_is_a_cuda_error(cuda_available):
    if cuda_available:
        pytest.skip("a device is present")
    L = harp.lib()
    h = ctypes.c_void_p()
    rad = (ctypes.c_int32 * 2)(16, 16)
    blk = np.zeros((16, 16, 16), np.float32)
    ptrs = (ctypes.POINTER(ctypes.c_float) * 2)(*(blk.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),) * 2)
    assert L.harp_plan_create(ctypes.byref(h), 256, 2, rad, ptrs, None, None) == 6
    assert not h.value


def test_codebook_checks_and_tables():
    with pytest.raises(harp.HarpError) as e:
        harp.Codebook("lloyd_max", 6, 128)
    assert e.value.status == 3
    with pytest.raises(harp.HarpError) as e:
        harp.Codebook("absmax", 1, 128)
    assert e.value.status == 3
    with pytest.raises(harp.HarpError) as e:
        harp.Codebook("lloyd_max", 3, 100)       # group not a multiple of 32
    assert e.value.status == 3
    with pytest.raises(harp.HarpError) as e:
        harp.Codebook("lloyd_max", 2, 128, centroids=[1.0, 0.5, 2.0, 3.0])
    assert e.value.status == 1
    cb = harp.Codebook("absmax", 4, 128)
    c, _ = cb.tables()
    np.testing.assert_array_equal(c, np.arange(16) - 8)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_library_lloyd_max_table_equals_oracle(bits):
    """The library solves the Lloyd-Max conditions itself (positive half,
    different start); its fp32 table must be the oracle's rounded table."""
    lib_c = harp.lloyd_max_centroids(bits)
    orc_c, _ = oracle.lloyd_max(bits)
    np.testing.assert_array_equal(lib_c, orc_c.astype(np.float32))
    cb = harp.Codebook("lloyd_max", bits, 128)
    c, t = cb.tables()
    np.testing.assert_array_equal(c, lib_c)
    mid = (0.5 * (lib_c[:-1].astype(np.float64) + lib_c[1:].astype(np.float64))).astype(np.float32)
    np.testing.assert_array_equal(t, mid)


@pytest.mark.parametrize("kind,b", [("hadamard", 16), ("hadamard", 5), ("qr", 16), ("qr", 43),
                                    ("qr", 7), ("cayley_hadamard", 8), ("cayley_hadamard", 2),
                                    ("cayley_hadamard", 3)])
def test_library_blocks_match_oracle_blocks(kind, b):
    """Same raw draws, two independent constructions (Householder vs
    Gram-Schmidt QR, Gauss-Jordan vs elimination Cayley, popcount vs doubling
    Sylvester): float32 blocks equal the oracle's float64 blocks to rounding."""
    n = 6
    g = synth.normal(17, 1, n * b * b).reshape(n, b, b)
    base = synth.normal(17, 2, b * b).reshape(b, b)
    lb = harp.stage_blocks(kind, b, n, g, base, 0.05)
    ob = oracle.stage_blocks(kind, b, n, g, base, 0.05)
    np.testing.assert_allclose(lb.astype(np.float64), ob, atol=4e-7, rtol=0)
    assert np.max(np.abs(lb.astype(np.float64) - ob)) <= 2.0 ** -24 * 2


def test_stage_blocks_argument_checks():
    with pytest.raises(harp.HarpError) as e:
        harp.stage_blocks("qr", 65, 1, np.zeros((1, 65, 65)))
    assert e.value.status == 3
    with pytest.raises(harp.HarpError) as e:
        harp.stage_blocks("qr", 4, 1, None)
    assert e.value.status == 1
    with pytest.raises(harp.HarpError) as e:
        harp.stage_blocks("hadamard", 5, 1, None, None)   # needs the base Gaussian
    assert e.value.status == 1
    with pytest.raises(harp.HarpError) as e:
        harp.stage_blocks("qr", 3, 1, np.zeros((1, 3, 3)))  # singular
    assert e.value.status == 2


def test_compute_calls_reject_bad_arguments_before_launch():
    L = harp.lib()
    # NULL plan / codebook
    assert L.harp_rotate(None, 0, 0, None, 0, None, 0, 4, 4, 4, 4, None) == 1
    assert L.harp_quantize(None, None, 0, 1, 128, 128, None, None, None) == 1
    assert L.harp_rotate_quantize(None, None, None, None, 0, 1, 128, None, None, None, None, 0, None) == 1
    assert L.harp_dequantize_unrotate(None, None, None, None, None, 1, 128, None, 0, None, 0, None) == 1
    cb = harp.Codebook("lloyd_max", 4, 128)
    # cols not a multiple of the group
    fake = ctypes.c_void_p(4096)
    assert L.harp_quantize(cb.handle, fake, 0, 1, 200, 200, fake, fake, None) == 2
    # misaligned pointer
    assert L.harp_quantize(cb.handle, ctypes.c_void_p(4100), 0, 1, 128, 128, fake, fake, None) == 4
    # leading dimension too small
    assert L.harp_quantize(cb.handle, fake, 0, 2, 128, 64, fake, fake, None) == 2
    # timing hook and pass count argument checks
    assert L.harp_set_pass_events(None, -1) == 1
    assert L.harp_set_pass_events(None, 3) == 1
    assert L.harp_set_pass_events(None, 0) == 0
    assert L.harp_pass_count(None, None, None, None) == 1
    assert L.harp_pass_fma(None, None, None, 0, None) == 1
    n = ctypes.c_size_t()
    assert L.harp_workspace_size(None, None, 10, 20, ctypes.byref(n)) == 0 and n.value == 0
    assert L.harp_workspace_size(ctypes.c_void_p(8), None, 10, 20, ctypes.byref(n)) == 0 and n.value == 1600


def test_host_buffer_calls_scratch_size_and_checks():
    """The host-buffer variants: scratch = values + codes + scales (+ the
    two-sided workspace), each part 256-byte aligned; argument errors come
    back before anything is copied or launched."""
    L = harp.lib()
    cb = harp.Codebook("lloyd_max", 3, 128)
    fake = ctypes.c_void_p(8)
    n = ctypes.c_size_t()
    # right-only, bf16 values: 64*256*2 + 64*256*3/8 + 64*2*2 bytes
    assert L.harp_host_scratch_size(None, fake, cb.handle, 64, 256, harp.HARP_BF16, ctypes.byref(n)) == 0
    assert n.value == 32768 + 6144 + 256
    # two-sided, fp32 values: plus rows*cols*8 bytes of workspace
    assert L.harp_host_scratch_size(fake, fake, cb.handle, 64, 256, harp.HARP_F32, ctypes.byref(n)) == 0
    assert n.value == 65536 + 6144 + 256 + 131072
    assert L.harp_host_scratch_size(None, None, cb.handle, 64, 256, harp.HARP_BF16, ctypes.byref(n)) == 1
    assert L.harp_host_scratch_size(None, fake, cb.handle, 64, 256, 2, ctypes.byref(n)) == 1   # f16 values
    assert L.harp_host_scratch_size(None, fake, cb.handle, 64, 256, harp.HARP_BF16, None) == 1
    # empty: nothing to do; missing or short scratch; missing host buffers
    assert L.harp_rotate_quantize_host(None, fake, cb.handle, None, harp.HARP_BF16, 0, 256, None, None,
                                       None, 0, None) == 0
    assert L.harp_rotate_quantize_host(None, fake, cb.handle, fake, harp.HARP_BF16, 64, 256, fake, fake,
                                       None, 0, None) == 5
    assert L.harp_rotate_quantize_host(None, fake, cb.handle, fake, harp.HARP_BF16, 64, 256, fake, fake,
                                       ctypes.c_void_p(4096), 1024, None) == 5
    assert L.harp_rotate_quantize_host(None, fake, cb.handle, None, harp.HARP_BF16, 64, 256, fake, fake,
                                       ctypes.c_void_p(4096), 1 << 20, None) == 1
    assert L.harp_dequantize_unrotate_host(None, fake, cb.handle, fake, fake, 64, 256, None, harp.HARP_BF16,
                                           ctypes.c_void_p(4096), 1 << 20, None) == 1
    assert L.harp_dequantize_unrotate_host(None, fake, cb.handle, fake, fake, 64, 256, fake, harp.HARP_F16,
                                           ctypes.c_void_p(4096), 1 << 20, None) == 1


def test_theta_calls_reject_bad_arguments_before_launch():
    L = harp.lib()
    fake = ctypes.c_void_p(4096)
    # radix outside [1, 64]
    assert L.harp_theta_blocks(65, 1, fake, 0.01, None, fake, None) == 3
    assert L.harp_theta_blocks(0, 1, fake, 0.01, None, fake, None) == 3
    # missing parameters, output or base mixer (b = 5 is not a power of two)
    assert L.harp_theta_blocks(4, 1, None, 0.01, None, fake, None) == 1
    assert L.harp_theta_blocks(4, 1, fake, 0.01, None, None, None) == 1
    assert L.harp_theta_blocks(5, 1, fake, 0.01, None, fake, None) == 1
    # non-finite scale, negative group count
    assert L.harp_theta_blocks(4, 1, fake, float("nan"), None, fake, None) == 1
    assert L.harp_theta_blocks(4, 1, fake, float("inf"), None, fake, None) == 1
    assert L.harp_theta_blocks(4, -1, fake, 0.01, None, fake, None) == 1
    # misaligned output or base
    assert L.harp_theta_blocks(4, 1, fake, 0.01, None, ctypes.c_void_p(4098), None) == 4
    assert L.harp_theta_blocks(5, 1, fake, 0.01, ctypes.c_void_p(4098), fake, None) == 4
    # no groups: nothing to do, no launch
    assert L.harp_theta_blocks(4, 0, None, 0.01, None, None, None) == 0
    # NULL plan
    assert L.harp_plan_load_theta(None, 0, fake, 0.01, None, None) == 1
    # two-stage codec: NULL plan or codebooks
    assert L.harp_requantize(None, None, None, None, 1, 128, 2, None, None, None, None, None) == 1
