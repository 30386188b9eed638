"""harp_rotate_quantize_static: the two-sided forward path for callers that
cannot allocate device memory (a host framework that owns every device byte,
a latency-critical path that must not call cudaMalloc). Its fp32
intermediate lives in a device array inside the library instead of a
caller-supplied workspace.

The checks go through the C ABI: two calls in a row of the static variant
must give what harp_rotate_quantize with an ordinary workspace gives (codes
and scales identical, the rotated copy within the fp32 tolerance), and a
matrix whose intermediate exceeds the array is refused before any launch.
This file is named so that pytest collects it last.
"""

import numpy as np
import pytest

import rotation_preconditioned_bit_b200 as harp
from rotation_preconditioned_bit_b200 import synth
from parity import TOL_F32, rel_l2

pytestmark = pytest.mark.gpu


def _case(rows_radix, cols_radix, bits, group, seed):
    import torch
    torch.cuda.set_device(0)
    left_s = synth.side_draws(seed, rows_radix, "qr", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(seed, cols_radix, "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    rows, cols = int(np.prod(rows_radix)), int(np.prod(cols_radix))
    W = synth.small_matrix(seed + 1, rows, cols, outlier_cols=4, scale=0.02)
    xb = torch.from_numpy(synth.to_bf16_bits(W).view(np.int16)).view(torch.bfloat16).cuda()
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    cb = harp.Codebook("lloyd_max", bits, group)
    return left, right, cb, xb


def test_static_workspace_matches_caller_workspace_twice():
    import torch
    torch.cuda.set_device(0)
    # 1024 x 2048 two-sided: a 16 MiB workspace need, inside the 32 MiB array
    left, right, cb, x = _case((16, 8, 8), (16, 16, 8), 4, 128, 31)
    rows, cols = x.shape
    assert harp.workspace_size(left, right, rows, cols) <= harp.HARP_STATIC_WORKSPACE_BYTES

    ref_codes, ref_scales = harp.empty_codes(rows, cols, cb)
    ref_rot = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ws = harp.empty_workspace(left, right, rows, cols)
    harp.harp_rotate_quantize(left, right, cb, x, ref_codes, ref_scales, ref_rot, ws)
    torch.cuda.synchronize()
    ref_codes, ref_scales, ref_rot = ref_codes.cpu(), ref_scales.cpu(), ref_rot.cpu().numpy()

    for _ in range(2):
        codes, scales = harp.empty_codes(rows, cols, cb)
        codes.fill_(0xA5)
        rot = torch.full((rows, cols), float("nan"), dtype=torch.float32, device="cuda")
        harp.harp_rotate_quantize_static(left, right, cb, x, codes, scales, rot)
        torch.cuda.synchronize()
        assert torch.equal(codes.cpu(), ref_codes)
        assert torch.equal(scales.cpu(), ref_scales)
        assert rel_l2(rot.cpu().numpy(), ref_rot) <= TOL_F32


def test_static_workspace_five_bit_codes_match_twice():
    """5-bit (PolarQuant Q5) codes take the whole-vector kernels, which write
    the same library array through another path: two calls in a row match
    the caller-workspace call."""
    import torch
    left, right, cb, x = _case((16, 8, 8), (8, 8, 16), 5, 128, 41)
    rows, cols = x.shape
    assert harp.workspace_size(left, right, rows, cols) <= harp.HARP_STATIC_WORKSPACE_BYTES
    ref_codes, ref_scales = harp.empty_codes(rows, cols, cb)
    ws = harp.empty_workspace(left, right, rows, cols)
    harp.harp_rotate_quantize(left, right, cb, x, ref_codes, ref_scales, None, ws)
    torch.cuda.synchronize()
    for _ in range(2):
        codes, scales = harp.empty_codes(rows, cols, cb)
        codes.fill_(0x5A)
        harp.harp_rotate_quantize_static(left, right, cb, x, codes, scales, None)
        torch.cuda.synchronize()
        assert torch.equal(codes.cpu(), ref_codes.cpu())
        assert torch.equal(scales.cpu(), ref_scales.cpu())


def test_static_workspace_rejects_oversized_matrix():
    # 4096 x 4096 needs a 128 MiB workspace: refused before any pointer is
    # used. The data pointers are NULL, so a reordering of the checks would
    # surface as HARP_ERR_INVALID_ARG, never as a launch.
    left, right, cb, _ = _case((16, 16, 16), (16, 16, 16), 2, 128, 5)
    assert harp.workspace_size(left, right, 4096, 4096) > harp.HARP_STATIC_WORKSPACE_BYTES
    st = harp.lib().harp_rotate_quantize_static(left.handle, right.handle, cb.handle, None,
                                                harp.HARP_BF16, 4096, 4096, None, None, None,
                                                None)
    assert st == 5  # HARP_ERR_WORKSPACE
