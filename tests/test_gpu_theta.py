"""Stage blocks built on the device from int8-stored parameters (HARP section
2.2, B = Q(theta) G_b with Givens for b = 2 and Cayley for b > 2; section 2.4,
int8 parameter storage), against the float64 oracle, through the C ABI.

Blocks: the device computes in double precision and rounds once to float, the
oracle in float64 with its own elimination order; the two float results may
differ only where the float64 values straddle a float rounding boundary, so
every entry must agree within one float ulp and almost all exactly.
Processors loaded this way must then rotate and quantize like the oracle's
processor built from the oracle's blocks (rounded to float, as the library
stores them).
"""

import numpy as np
import pytest

import oracle
from parity import TOL_F32, compare_quant, rel_l2
from rotation_preconditioned_bit_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import rotation_preconditioned_bit_b200 as harp

SCALE = np.float32(0.05 / 40)     # stored values spread ~40 steps: theta ~ 0.05 N(0,1)


def base_mixer(b, seed):
    """A fixed orthogonal float32 G_b for b not a power of two (None else)."""
    if (b & (b - 1)) == 0:
        return None
    g = synth.normal(seed, synth.S_BASE_R, b * b).reshape(b, b)
    q, r = np.linalg.qr(g)
    return (q * np.sign(np.diag(r))).astype(np.float32)


def oracle_blocks_f32(b, q, G):
    return oracle.theta_blocks(b, q, SCALE, None if G is None else G.astype(np.float64)).astype(np.float32)


def assert_blocks_match(got, want_f64):
    want = want_f64.astype(np.float32)
    ulp = np.spacing(np.abs(want)).astype(np.float64)
    diff = np.abs(got.astype(np.float64) - want.astype(np.float64))
    assert np.all(diff <= ulp), f"max diff {diff.max()} over one ulp"
    assert np.mean(got == want) >= 0.999


@pytest.mark.parametrize("b,n_groups", [(1, 7), (2, 3000), (3, 50), (5, 333), (7, 64), (8, 1300),
                                        (16, 1500), (32, 40), (43, 9), (64, 5)])
def test_theta_blocks_match_oracle(b, n_groups):
    torch.cuda.set_device(0)
    q = synth.theta_draws(40 + b, 0, n_groups, b)
    G = base_mixer(b, 40 + b)
    want = oracle.theta_blocks(b, q, SCALE, None if G is None else G.astype(np.float64))
    out = torch.full((n_groups, b, b), float("nan"), dtype=torch.float32, device="cuda")
    qt = torch.from_numpy(q).cuda() if q.size else None
    gt = None if G is None else torch.from_numpy(G).cuda()
    harp.harp_theta_blocks(b, qt, SCALE, out, gt)
    torch.cuda.synchronize()
    assert_blocks_match(out.cpu().numpy(), want)


@pytest.mark.parametrize("b", [2, 8, 16, 64])
def test_theta_zero_gives_the_sylvester_mixer_exactly(b):
    p = max(b * (b - 1) // 2, 1)
    out = torch.empty((11, b, b), dtype=torch.float32, device="cuda")
    harp.harp_theta_blocks(b, torch.zeros((11, p), dtype=torch.int8, device="cuda"), SCALE, out)
    i = np.arange(b)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    H = (np.where(pc % 2 == 0, 1.0, -1.0) / np.sqrt(b)).astype(np.float32)
    assert np.array_equal(out.cpu().numpy(), np.broadcast_to(H, (11, b, b)))


def _theta_side(seed, radix, stage0):
    """Per stage: (int8 parameters, base mixer) for a processor of `radix`."""
    d = int(np.prod(radix))
    return [(synth.theta_draws(seed, stage0 + t, d // b, b), base_mixer(b, seed + t))
            for t, b in enumerate(radix)]


def _load(plan, params):
    for t, (q, G) in enumerate(params):
        harp.harp_plan_load_theta(plan, t, torch.from_numpy(q).cuda() if q.size else None, SCALE,
                                  None if G is None else torch.from_numpy(G).cuda())


def _oracle_processor(radix, params, signs):
    blocks = [oracle_blocks_f32(b, q, G).astype(np.float64) for b, (q, G) in zip(radix, params)]
    return oracle.Processor(radix, blocks, signs.astype(np.float64))


def test_loaded_plans_rotate_and_quantize_like_the_oracle():
    """Plans created with Hadamard blocks, then every stage replaced on the
    device from int8 parameters: the two-sided forward rotation + 3-bit
    Lloyd-Max, its inverse, and both one-sided rotations match the oracle's
    processor built from its own blocks. Radices 2 (Givens), 5 and 16 / 8
    (Cayley over a QR / Sylvester base mixer)."""
    torch.cuda.set_device(0)
    lrad, rrad = (2, 16, 16), (5, 16, 8)
    rows, cols = 512, 640
    left_s = synth.side_draws(61, lrad, "hadamard", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(61, rrad, "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    lp, rp = _theta_side(62, lrad, 0), _theta_side(63, rrad, 10)
    _load(left, lp)
    _load(right, rp)
    Pl = _oracle_processor(lrad, lp, left_s.signs)
    Pr = _oracle_processor(rrad, rp, right_s.signs)

    W = synth.small_matrix(64, rows, cols, outlier_cols=5, scale=0.02)
    Wb = synth.to_bf16_bits(W)
    X = synth.bf16_bits_to_f64(Wb)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(X, Pl, Pr, "lloyd_max", 3, 128)
    cb = harp.Codebook("lloyd_max", 3, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(left, right, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16), oc, osc, m, sm, 3, 128)

    raw, sc = synth.random_code_stream(65, rows, cols, 3, 128)
    ref_inv = oracle.dequantize_unrotate(oracle.unpack(3, raw, cols), sc, Pl, Pr, "lloyd_max", 3, 128)
    out = harp.dequantize_unrotate(left, right, cb, torch.from_numpy(raw).cuda(),
                                   torch.from_numpy(sc.view(np.int16)).cuda(), rows, cols, torch.float32)
    assert rel_l2(out.cpu().numpy(), ref_inv) <= TOL_F32

    # one-sided calls read the plan's other block layouts
    xf = torch.from_numpy(X.astype(np.float32)).cuda()
    o = torch.empty_like(xf)
    harp.harp_rotate(right, harp.HARP_RIGHT, harp.HARP_FWD, xf, o)
    assert rel_l2(o.cpu().numpy(), Pr.rotate_rows(X.astype(np.float32).astype(np.float64))) <= TOL_F32
    harp.harp_rotate(left, harp.HARP_LEFT, harp.HARP_INV, xf, o)
    assert rel_l2(o.cpu().numpy(),
                  Pl.rotate_cols(X.astype(np.float32).astype(np.float64), inverse=True)) <= TOL_F32


def test_loaded_plan_feeds_the_row_kernel():
    """A right-only rotate + quantize whose radices (16, 8, 4) take the row
    kernel, which reads the plan's group-interleaved copy of the forward
    blocks: after every stage is replaced from int8 parameters, the rotated
    rows, codes and scales match the oracle's processor built from the same
    parameters."""
    torch.cuda.set_device(0)
    radix = (16, 8, 4)
    rows, cols = 300, 512
    side = synth.side_draws(81, radix, "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan = harp.Plan.from_side(side)
    params = _theta_side(82, radix, 20)
    _load(plan, params)
    P = _oracle_processor(radix, params, side.signs)
    W = synth.small_matrix(83, rows, cols, outlier_cols=3, scale=0.02)
    Wb = synth.to_bf16_bits(W)
    X = synth.bf16_bits_to_f64(Wb)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(X, None, P, "absmax", 4, 128)
    cb = harp.Codebook("absmax", 4, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16), oc, osc, m, sm, 4, 128)


def test_load_is_stream_ordered_and_rejects_bad_stage():
    """A rotation launched before a load on the same stream sees the old
    blocks, one launched after it the new ones; a stage outside [0, m) is an
    argument error."""
    torch.cuda.set_device(0)
    radix = (16, 16)
    s = synth.side_draws(71, radix, "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan = harp.Plan.from_side(s)
    X = synth.small_matrix(72, 64, 256)
    xf = torch.from_numpy(X.astype(np.float32)).cuda()
    before, after = torch.empty_like(xf), torch.empty_like(xf)
    params = _theta_side(73, radix, 0)
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_FWD, xf, before)
    _load(plan, params)
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_FWD, xf, after)
    Xf = X.astype(np.float32).astype(np.float64)
    assert rel_l2(before.cpu().numpy(), oracle.processor(s).rotate_rows(Xf)) <= TOL_F32
    P = _oracle_processor(radix, params, s.signs)
    assert rel_l2(after.cpu().numpy(), P.rotate_rows(Xf)) <= TOL_F32
    with pytest.raises(harp.HarpError) as e:
        harp.harp_plan_load_theta(plan, 2, torch.zeros((16, 120), dtype=torch.int8, device="cuda"), SCALE)
    assert e.value.status == 1
