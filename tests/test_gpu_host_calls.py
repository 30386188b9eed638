"""The host-buffer variants of the fused calls (harp_rotate_quantize_host,
harp_dequantize_unrotate_host) against the device calls they wrap: same
kernels, so the codes, scales and restored values must agree exactly, for a
two-sided processor (pass kernels) and a right-only one (row kernel)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from rotation_preconditioned_bit_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


import rotation_preconditioned_bit_b200 as harp  # noqa: E402


@pytest.mark.parametrize("two_sided", [True, False])
def test_host_calls_match_device_calls(two_sided):
    rows, cols = 512, 256
    right = harp.Plan.from_side(synth.side_draws(121, (16, 16), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R))
    left = (harp.Plan.from_side(synth.side_draws(122, (8, 8, 8), "qr", synth.S_SIGNS_L, synth.S_BLOCKS_L))
            if two_sided else None)
    cb = harp.Codebook("lloyd_max", 4, 128)
    Wb = synth.to_bf16_bits(synth.small_matrix(123, rows, cols, outlier_cols=2, scale=0.02))
    x_host = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = x_host.cuda()
    ws = harp.empty_workspace(left, right, rows, cols) if left else None
    codes_d, scales_d = harp.empty_codes(rows, cols, cb)
    harp.harp_rotate_quantize(left, right, cb, x, codes_d, scales_d, None, ws)
    out_d = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    harp.harp_dequantize_unrotate(left, right, cb, codes_d, scales_d, out_d, ws)

    scratch = harp.empty_host_scratch(left, right, cb, rows, cols, harp.HARP_BF16)
    codes_h = torch.empty(codes_d.shape, dtype=codes_d.dtype).pin_memory()
    scales_h = torch.empty(scales_d.shape, dtype=scales_d.dtype).pin_memory()
    out_h = torch.empty((rows, cols), dtype=torch.bfloat16).pin_memory()
    harp.harp_rotate_quantize_host(left, right, cb, x_host, codes_h, scales_h, scratch)
    harp.harp_dequantize_unrotate_host(left, right, cb, codes_h, scales_h, out_h, scratch)
    torch.cuda.synchronize()
    assert torch.equal(codes_h, codes_d.cpu())
    assert torch.equal(scales_h, scales_d.cpu())
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))

    small = torch.empty(scratch.numel() - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(harp.HarpError) as e:
        harp.harp_rotate_quantize_host(left, right, cb, x_host, codes_h, scales_h, small)
    assert e.value.status == 5
