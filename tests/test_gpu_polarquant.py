"""PolarQuant's per-block workload and two-stage codec on the GPU, against the
float64 oracle, through the C ABI.

PolarQuant (gist.science paper 2603.29078) section 2 cuts every weight row
into blocks of d = 128, rotates each block by the Walsh-Hadamard matrix H_128
after normalising it, and codes the N(0,1)-scaled coordinates with Lloyd-Max
centroids; section 3 uses 5-bit codes (Q5) and, as a pre-processing step,
hands the restored FP16 weights to an absmax INT4 quantizer. Here a block of
128 is a row of the matrix viewed as [rows * cols / 128, 128], the rotation is
a right-side processor of radices (16, 8) with normalised Sylvester blocks
and no signs (exactly H_128), and the group scale is the block's RMS.
"""

import numpy as np
import pytest

import oracle
from parity import TOL_F32, compare_quant, np_unpack, rel_l2
from rotation_preconditioned_bit_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import rotation_preconditioned_bit_b200 as harp

RADIX = (16, 8)


def h128_plans():
    d = int(np.prod(RADIX))
    lib_blocks = [harp.stage_blocks("hadamard", b, d // b) for b in RADIX]
    orc_blocks = [oracle.stage_blocks("hadamard", b, d // b) for b in RADIX]
    return harp.Plan(RADIX, lib_blocks), oracle.Processor(RADIX, orc_blocks)


def bf16_matrix(seed, rows, cols):
    W = synth.student_t(seed, 3, rows * cols).reshape(rows, cols) * 0.02
    W[:, synth.choose(seed, synth.S_OUTLIER, cols, max(1, cols // 200))] *= 20.0
    return synth.to_bf16_bits(W)


def scales_np(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("rows,cols", [(64, 1024), (4096, 4096)])
def test_per_block_q5_forward_and_inverse(rows, cols):
    """Forward: rows of 128 rotated by H_128, 5-bit Lloyd-Max with the block
    RMS as scale; inverse: dequantise and rotate back. The 4096 x 4096 case
    is the benchmark's shape and launch configuration."""
    torch.cuda.set_device(0)
    plan, P = h128_plans()
    Wb = bf16_matrix(80 + rows, rows, cols)
    n = rows * cols // 128
    X = synth.bf16_bits_to_f64(Wb).reshape(n, 128)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(X, None, P, "lloyd_max", 5, 128)
    cb = harp.Codebook("lloyd_max", 5, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda().view(n, 128)
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, 5, 128)
    # the codes viewed as [rows, cols * 5 / 8] are the same bytes: one row of
    # the weight holds cols / 128 consecutive blocks
    assert codes.view(rows, cols * 5 // 8).is_contiguous()
    back = harp.dequantize_unrotate(None, plan, cb, codes, scales, n, 128, torch.float32)
    ref_back = oracle.dequantize_unrotate(np_unpack(codes.cpu().numpy(), 5, 128), scales_np(scales),
                                          None, P, "lloyd_max", 5, 128)
    assert rel_l2(back.cpu().numpy(), ref_back) <= TOL_F32


def _requant_case(plan, P, rows, d, mid, seed, kind_in="lloyd_max", bits_in=5):
    raw, sc = synth.random_code_stream(seed, rows, d, bits_in, 128)
    cb_in = harp.Codebook(kind_in, bits_in, 128)
    cb_out = harp.Codebook("absmax", 4, 128)
    codes_out, scales_out = harp.empty_codes(rows, d, cb_out)
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[mid]
    restored = torch.empty((rows, d), dtype=dt, device="cuda")
    harp.harp_requantize(plan, cb_in, torch.from_numpy(raw).cuda(), torch.from_numpy(sc.view(np.int16)).cuda(),
                         rows, d, mid, cb_out, codes_out, scales_out, restored)
    torch.cuda.synchronize()
    Y, oc, _, osc, _, _ = oracle.requantize(oracle.unpack(bits_in, raw, d), sc, P, kind_in, bits_in, 128,
                                            mid, "absmax", 4, 128)
    got = restored.float().cpu().numpy().astype(np.float64)
    return got, Y, codes_out, scales_out


def assert_restored_match(got, Y, mid):
    """16-bit restored weights: the GPU rounds its fp32 rotation, the oracle
    its float64 one, so a value may land one unit of the 16-bit type away
    where the two straddle a rounding boundary, or a little further for a
    value far below its row's size (fp32 rounding error is relative to the
    row, not to the value)."""
    if mid == "f16":
        ulp = np.spacing(np.abs(Y).astype(np.float16)).astype(np.float64)
    else:
        ulp = np.spacing(np.abs(Y).astype(np.float32)).astype(np.float64) * 65536
    row = np.linalg.norm(Y, axis=1, keepdims=True)
    assert np.all(np.abs(got - Y) <= np.maximum(ulp, 1e-6 * row))
    assert np.mean(got == Y) > 0.999


@pytest.mark.parametrize("mid", ["f16", "bf16", "f32"])
def test_requantize_q5_to_int4_absmax(mid):
    """The fused two-stage codec: the restored weights agree with the
    oracle's within one unit of the storage type (almost all exactly), and
    the INT4 absmax codes and scales are exactly what the oracle's quantizer
    gives for those restored weights."""
    torch.cuda.set_device(0)
    plan, P = h128_plans()
    rows = 3000
    got, Y, codes_out, scales_out = _requant_case(plan, P, rows, 128, mid, 90)
    if mid == "f32":
        assert rel_l2(got, Y) <= TOL_F32
    else:
        assert_restored_match(got, Y, mid)
    oc, osc, m, sm = oracle.quantize("absmax", 4, 128, got)
    compare_quant(codes_out.cpu().numpy(), scales_np(scales_out), oc, osc, m, sm, 4, 128)


def test_requantize_general_processor_and_absmax_input():
    """A random orthogonal (16, 8, 8) row processor with signs, 3-bit absmax
    first stage, bf16 restored weights: the same two checks."""
    torch.cuda.set_device(0)
    side = synth.side_draws(95, (16, 8, 8), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan, P = harp.Plan.from_side(side), oracle.processor(side)
    got, Y, codes_out, scales_out = _requant_case(plan, P, 257, 1024, "bf16", 96, "absmax", 3)
    assert_restored_match(got, Y, "bf16")
    oc, osc, m, sm = oracle.quantize("absmax", 4, 128, got)
    compare_quant(codes_out.cpu().numpy(), scales_np(scales_out), oc, osc, m, sm, 4, 128)


def test_requantize_argument_checks():
    torch.cuda.set_device(0)
    plan, _ = h128_plans()
    cb5, cb4 = harp.Codebook("lloyd_max", 5, 128), harp.Codebook("absmax", 4, 128)
    c = torch.zeros((4, 80), dtype=torch.uint8, device="cuda")
    s = torch.zeros((4, 1), dtype=torch.int16, device="cuda")
    co = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(harp.HarpError) as e:           # cols != plan's d
        harp.harp_requantize(plan, cb5, c, s, 4, 256, "f16", cb4, co, s)
    assert e.value.status == 2
    L = harp.lib()
    assert L.harp_requantize(plan.handle, cb5.handle, None, None, 4, 128, 7, None, cb4.handle,
                             None, None, None) == 1       # bad storage type
    assert L.harp_requantize(plan.handle, cb5.handle, None, None, 0, 128, 2, None, cb4.handle,
                             None, None, None) == 0       # empty: nothing to do


def test_two_sided_q5_takes_the_whole_vector_path():
    """5-bit codes on both sides of a 512 x 1024 weight (the pass kernels
    handle 2-4 bits; 5 bits run column pass + row pass): forward and inverse
    against the oracle."""
    torch.cuda.set_device(0)
    left_s = synth.side_draws(97, (8, 8, 8), "qr", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(97, (16, 8, 8), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    Pl, Pr = oracle.processor(left_s), oracle.processor(right_s)
    cb = harp.Codebook("lloyd_max", 5, 128)
    assert harp.harp_pass_count(left, right, cb) == 0
    Wb = bf16_matrix(98, 512, 1024)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.bf16_bits_to_f64(Wb), Pl, Pr, "lloyd_max", 5, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(left, right, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, 5, 128)
    back = harp.dequantize_unrotate(left, right, cb, codes, scales, 512, 1024, torch.float32)
    ref_back = oracle.dequantize_unrotate(np_unpack(codes.cpu().numpy(), 5, 1024), scales_np(scales),
                                          Pl, Pr, "lloyd_max", 5, 128)
    assert rel_l2(back.cpu().numpy(), ref_back) <= TOL_F32


def test_short_vectors_mixed_sylvester_and_random_stages():
    """A d = 128 right processor whose first stage is all-Sylvester (the
    butterfly) and whose second has random orthogonal blocks (FMAs), with
    signs: the general build of the short-vector kernel runs both stage
    kinds; forward with the rotated copy and the inverse, against the
    oracle's processor built from its own blocks of the same draws."""
    torch.cuda.set_device(0)
    radix, d, rows = (8, 16), 128, 300
    g = synth.normal(111, 5, (d // 16) * 16 * 16).reshape(d // 16, 16, 16)
    signs = synth.signs(112, 3, d)
    plan = harp.Plan(radix, [harp.stage_blocks("hadamard", 8, d // 8), harp.stage_blocks("qr", 16, d // 16, gauss=g)],
                     signs)
    P = oracle.Processor(radix, [oracle.stage_blocks("hadamard", 8, d // 8),
                                 oracle.stage_blocks("qr", 16, d // 16, gauss=g)], signs.astype(np.float64))
    Wb = bf16_matrix(113, rows, d)
    X = synth.bf16_bits_to_f64(Wb)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(X, None, P, "lloyd_max", 4, 128)
    cb = harp.Codebook("lloyd_max", 4, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, 4, 128)
    back = harp.dequantize_unrotate(None, plan, cb, codes, scales, rows, d, torch.float32)
    ref_back = oracle.dequantize_unrotate(np_unpack(codes.cpu().numpy(), 4, d), scales_np(scales),
                                          None, P, "lloyd_max", 4, 128)
    assert rel_l2(back.cpu().numpy(), ref_back) <= TOL_F32


@pytest.mark.parametrize("radix,bits,group", [((4, 8), 4, 32), ((8, 8), 3, 64), ((2, 16, 4), 2, 32)])
def test_short_vectors_all_three_calls(radix, bits, group):
    """Rows of 32, 64 and 128 coordinates (one thread per row in the
    short-vector kernel), 1000 rows (a ragged last tile of 256), random
    orthogonal blocks with signs: forward (bf16 in, fp32 rotated copy),
    inverse to bf16, and the two-stage codec to 4-bit absmax."""
    torch.cuda.set_device(0)
    side = synth.side_draws(101 + bits, radix, "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan, P = harp.Plan.from_side(side), oracle.processor(side)
    d, rows = int(np.prod(radix)), 1000
    Wb = bf16_matrix(102 + bits, rows, d)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.bf16_bits_to_f64(Wb), None, P, "lloyd_max", bits, group)
    cb = harp.Codebook("lloyd_max", bits, group)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
    raw, sc = synth.random_code_stream(103, rows, d, bits, group)
    ref_inv = oracle.dequantize_unrotate(oracle.unpack(bits, raw, d), sc, None, P, "lloyd_max", bits, group)
    out = harp.dequantize_unrotate(None, plan, cb, torch.from_numpy(raw).cuda(),
                                   torch.from_numpy(sc.view(np.int16)).cuda(), rows, d, torch.bfloat16)
    assert rel_l2(out.float().cpu().numpy(), ref_inv) <= 1e-2
    got, Y, codes_out, scales_out = _requant_case_g(plan, P, raw, sc, rows, d, bits, group)
    assert_restored_match(got, Y, "f16")
    oc2, osc2, m2, sm2 = oracle.quantize("absmax", 4, 32, got)
    compare_quant(codes_out.cpu().numpy(), scales_np(scales_out), oc2, osc2, m2, sm2, 4, 32)


def _requant_case_g(plan, P, raw, sc, rows, d, bits, group):
    cb_in = harp.Codebook("lloyd_max", bits, group)
    cb_out = harp.Codebook("absmax", 4, 32)
    codes_out, scales_out = harp.empty_codes(rows, d, cb_out)
    restored = torch.empty((rows, d), dtype=torch.float16, device="cuda")
    harp.harp_requantize(plan, cb_in, torch.from_numpy(raw).cuda(), torch.from_numpy(sc.view(np.int16)).cuda(),
                         rows, d, "f16", cb_out, codes_out, scales_out, restored)
    torch.cuda.synchronize()
    Y = oracle.requantize(oracle.unpack(bits, raw, d), sc, P, "lloyd_max", bits, group, "f16", "absmax", 4, 32)[0]
    return restored.float().cpu().numpy().astype(np.float64), Y, codes_out, scales_out
