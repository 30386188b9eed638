"""GPU-vs-oracle parity of the CUDA path, called through the C ABI.

Every input comes from the seeded generator (synth); the oracle builds its own
float64 blocks and codebook from the same raw draws. Full-size workloads are
compared element by element, forward and inverse, at every full size (the
oracle spreads its independent rows and columns over the host threads), in
the launch configuration the benchmark times.
"""

import numpy as np
import pytest

import oracle
from parity import TOL_BF16, TOL_F32, compare_quant, np_unpack, rel_l2
from rotation_preconditioned_bit_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import rotation_preconditioned_bit_b200 as harp


_WL = {}


def wl(name, **kw):
    key = (name, tuple(sorted(kw.items())))
    if key not in _WL:
        _WL[key] = synth.workload(name, **kw)
    return _WL[key]


def to_dev(w):
    if w.dtype == "bf16":
        return torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w.x)).cuda()


def scales_np(t):
    return t.cpu().numpy().view(np.uint16)


# ------------------------------------------------------------ 64 x 256 fp32, (16,16) Sylvester

def test_c1_rotate_matches_oracle():
    w = wl("c1")
    P = oracle.processor(w.right)
    ref = P.rotate_rows(synth.x_as_f64(w))
    plan = harp.Plan.from_side(w.right)
    x = to_dev(w)
    out = torch.empty_like(x)
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_FWD, x, out)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL_F32
    back = torch.empty_like(x)
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_INV, out, back)
    assert rel_l2(back.cpu().numpy(), synth.x_as_f64(w)) <= TOL_F32


def test_c1_rotate_quantize_matches_oracle():
    w = wl("c1")
    q = w.quants[0]
    P = oracle.processor(w.right)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.x_as_f64(w), None, P, q.kind, q.bits, q.group)
    plan = harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, to_dev(w), want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    rep = compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)
    assert rep["near_boundary"] < 0.001 * rep["elements"]


# ------------------------------------------------------------ 4096 x 4096 bf16, two-sided

@pytest.fixture(scope="module")
def c2_ref():
    w = wl("c2")
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    return w, Pr.rotate_rows(Pl.rotate_cols(synth.x_as_f64(w)))


@pytest.mark.parametrize("qi", [0, 1])
def test_c2_two_sided_full_matrix(c2_ref, qi):
    w, ref = c2_ref
    q = w.quants[qi]
    oc, osc, m, sm = oracle.quantize(q.kind, q.bits, q.group, ref)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    x = to_dev(w)
    codes, scales, rot = harp.rotate_quantize(left, right, cb, x, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    rep = compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)
    print(f"\nc2 {q.kind} {q.bits}-bit:", rep)
    # the benchmark's call (no fp32 copy) gives the same bytes
    codes2, scales2, _ = harp.rotate_quantize(left, right, cb, x)
    assert torch.equal(codes2, codes) and torch.equal(scales2, scales)


@pytest.fixture(params=["tc", "ffma"])
def block_stages(request):
    """Run a test with the two-sided calls' block stages forced to the tensor
    cores (tcgen05 3xTF32) or to fp32 FMAs; back to automatic afterwards."""
    mode = harp.HARP_BLOCK_STAGES_TC if request.param == "tc" else harp.HARP_BLOCK_STAGES_FFMA
    harp.harp_set_block_stages(mode)
    yield request.param
    harp.harp_set_block_stages(harp.HARP_BLOCK_STAGES_AUTO)


def test_c2_both_block_stage_kinds_match_oracle(c2_ref, block_stages):
    """The 4096 x 4096 workload through each block-stage implementation:
    forward (2- and 4-bit Lloyd-Max, rotated copy and codes) and the inverse
    of the oracle's own codes, every element against the oracle."""
    w, ref = c2_ref
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    x = to_dev(w)
    for q in w.quants:
        oc, osc, m, sm = oracle.quantize(q.kind, q.bits, q.group, ref)
        cb = harp.Codebook(q.kind, q.bits, q.group)
        codes, scales, rot = harp.rotate_quantize(left, right, cb, x, want_rotated=True)
        e = rel_l2(rot.cpu().numpy(), ref)
        del rot
        rep = compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)
        print(f"\nc2 {block_stages} {q.bits}-bit: rotated rel_l2 {e:.3e}", rep)
        assert e <= TOL_F32
        _inverse_full(w, left, right, q, oracle.pack(q.bits, oc), osc, Pl, Pr, f"c2 {block_stages} {q.bits}-bit")


def test_c2_unfused_matches_oracle_like_fused(c2_ref):
    """The separate calls (left rotation, right rotation, standalone
    quantizer) meet the same bar against the oracle as the fused call. The
    two paths run different kernels that sum in different orders, so their
    codes may differ only inside the boundary band, which compare_quant
    excludes and counts."""
    w, ref = c2_ref
    q = w.quants[1]
    oc, osc, m, sm = oracle.quantize(q.kind, q.bits, q.group, ref)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    x = to_dev(w)
    codes, scales, _ = harp.rotate_quantize(left, right, cb, x)
    t = torch.empty(x.shape, dtype=torch.float32, device="cuda")
    harp.harp_rotate(left, harp.HARP_LEFT, harp.HARP_FWD, x, t)
    t2 = torch.empty_like(t)
    harp.harp_rotate(right, harp.HARP_RIGHT, harp.HARP_FWD, t, t2)
    assert rel_l2(t2.cpu().numpy(), ref) <= TOL_F32
    c2, s2 = harp.empty_codes(*x.shape, cb)
    harp.harp_quantize(cb, t2, c2, s2)
    compare_quant(c2.cpu().numpy(), scales_np(s2), oc, osc, m, sm, q.bits, q.group)
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)


# ------------------------------------------------------------ [T, 4096] activations, per-token absmax

@pytest.mark.parametrize("T", [1, 16, 256, 8192])
def test_c3_activation_rows(T):
    w = wl("c3", tokens=T)
    q = w.quants[0]
    P = oracle.processor(w.right)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.x_as_f64(w), None, P, q.kind, q.bits, q.group)
    plan = harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    codes, scales, rot = harp.rotate_quantize(None, plan, cb, to_dev(w), want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)
    # bf16 rotated activations
    xb = torch.empty((T, 4096), dtype=torch.bfloat16, device="cuda")
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_FWD, to_dev(w), xb)
    assert rel_l2(xb.float().cpu().numpy(), ref) <= TOL_BF16


@pytest.mark.parametrize("radix,rows,dtype", [((16, 16, 16), 37, "f32"), ((4, 8, 16, 2, 8), 61, "bf16"),
                                              ((2, 4, 8, 16), 1000, "bf16"), ((16, 16), 9, "f32")])
@pytest.mark.parametrize("kind,bits,group", [("lloyd_max", 3, 128), ("absmax", 4, 256), ("lloyd_max", 2, 64)])
def test_row_kernel_shapes(radix, rows, dtype, kind, bits, group):
    """Right-only rotate + quantize of whole rows (the row kernel: radices 2, 4,
    8, 16) on ragged row counts, fp32 and bf16 inputs, several group sizes,
    with the fp32 rotated copy, against the oracle element by element."""
    d = int(np.prod(radix))
    if d % group:
        pytest.skip("group does not divide the row")
    s = synth.side_draws(90 + d, radix, "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    X = synth.small_matrix(91 + rows, rows, d, outlier_cols=3, scale=0.02)
    if dtype == "bf16":
        Xb = synth.to_bf16_bits(X)
        x = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
        Xf = synth.bf16_bits_to_f64(Xb)
    else:
        X32 = X.astype(np.float32)
        x = torch.from_numpy(X32).cuda()
        Xf = X32.astype(np.float64)
    P = oracle.processor(s)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(Xf, None, P, kind, bits, group)
    cb = harp.Codebook(kind, bits, group)
    codes, scales, rot = harp.rotate_quantize(None, harp.Plan.from_side(s), cb, x, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)


# ------------------------------------------------------------ inverse paths, whole matrices

def _inverse_full(w, left, right, q, raw, sc, Pl, Pr, label):
    """dequantize + unrotate of the packed code stream `raw` with fp16 scales
    `sc` (never produced by the CUDA path) against the oracle, every element,
    fp32 and bf16 outputs."""
    rows, cols = w.rows, w.cols
    ref = oracle.dequantize_unrotate(oracle.unpack(q.bits, raw, cols), sc, Pl, Pr, q.kind, q.bits, q.group)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    codes = torch.from_numpy(np.ascontiguousarray(raw)).cuda()
    scales = torch.from_numpy(np.ascontiguousarray(sc).view(np.int16)).cuda()
    out = harp.dequantize_unrotate(left, right, cb, codes, scales, rows, cols, torch.float32)
    e32 = rel_l2(out.cpu().numpy(), ref)
    del out
    outb = harp.dequantize_unrotate(left, right, cb, codes, scales, rows, cols, torch.bfloat16)
    e16 = rel_l2(outb.float().cpu().numpy(), ref)
    print(f"\n{label}: inverse rel_l2 fp32 {e32:.3e} bf16 {e16:.3e}")
    assert e32 <= TOL_F32
    assert e16 <= TOL_BF16
    return ref


@pytest.mark.parametrize("qi", [0, 1])
def test_c2_inverse_full_matrix(c2_ref, qi):
    """The benchmarked inverse: 4096 x 4096, (16,16,16) on both sides,
    2- and 4-bit Lloyd-Max g128, fp32 and bf16 outputs, every element --
    on a seeded random code stream and on the oracle forward's own codes
    (HARP section 5: the rotation is undone exactly by the transposes;
    PolarQuant section 2: dequantise, then rotate back)."""
    w, ref = c2_ref
    q = w.quants[qi]
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    raw, sc = synth.random_code_stream(2020 + qi, w.rows, w.cols, q.bits, q.group)
    _inverse_full(w, left, right, q, raw, sc, Pl, Pr, f"c2 {q.bits}-bit random stream")
    oc, osc, _, _ = oracle.quantize(q.kind, q.bits, q.group, ref, with_margins=False)
    _inverse_full(w, left, right, q, oracle.pack(q.bits, oc), osc, Pl, Pr, f"c2 {q.bits}-bit oracle codes")


# ------------------------------------------------------------ the large workloads, whole matrices

@pytest.fixture(scope="module")
def c4_ref():
    w = wl("c4")
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    return w, Pl, Pr, Pr.rotate_rows(Pl.rotate_cols(synth.x_as_f64(w)))


def _full_forward(w, Pl, Pr, ref, q, label):
    oc, osc, m, sm = oracle.quantize(q.kind, q.bits, q.group, ref)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    x = to_dev(w)
    codes, scales, rot = harp.rotate_quantize(left, right, cb, x, want_rotated=True)
    e = rel_l2(rot.cpu().numpy(), ref)
    del rot
    rep = compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, q.bits, q.group)
    print(f"\n{label}: rotated rel_l2 {e:.3e}", rep)
    assert e <= TOL_F32
    # the benchmark's call (no fp32 copy) gives the same bytes
    codes2, scales2, _ = harp.rotate_quantize(left, right, cb, x)
    assert torch.equal(codes2, codes) and torch.equal(scales2, scales)
    return left, right, cb, codes, scales, oc, osc


def test_c4_forward_full_and_round_trip(c4_ref):
    w, Pl, Pr, ref = c4_ref
    q = w.quants[0]
    left, right, cb, codes, scales, oc, osc = _full_forward(w, Pl, Pr, ref, q, "c4 3-bit")
    # round trip: an exact change of basis keeps the error norm
    What = harp.dequantize_unrotate(left, right, cb, codes, scales, w.rows, w.cols, torch.float32)
    Wp_hat = torch.empty((w.rows, w.cols), dtype=torch.float32, device="cuda")
    harp.harp_dequantize(cb, codes, scales, Wp_hat)
    x = to_dev(w).float()
    _, _, rot = harp.rotate_quantize(left, right, cb, to_dev(w), want_rotated=True)
    e_orig = torch.linalg.norm((x - What).double()).item()
    e_rot = torch.linalg.norm((rot - Wp_hat).double()).item()
    assert abs(e_orig - e_rot) <= 1e-5 * e_rot
    # the inverse of the oracle's own codes, every element
    _inverse_full(w, left, right, q, oracle.pack(q.bits, oc), osc, Pl, Pr, "c4 3-bit oracle codes")


def test_c4_inverse_full():
    w = wl("c4")
    q = w.quants[0]
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    raw, sc = synth.random_code_stream(4040, w.rows, w.cols, q.bits, q.group)
    _inverse_full(w, left, right, q, raw, sc, Pl, Pr, "c4 3-bit random stream")
    # the standalone dequantiser on the same bytes
    cb = harp.Codebook(q.kind, q.bits, q.group)
    Wp = oracle.dequantize(q.kind, q.bits, q.group, oracle.unpack(q.bits, raw, w.cols), sc)
    deq = torch.empty((w.rows, w.cols), dtype=torch.float32, device="cuda")
    harp.harp_dequantize(cb, torch.from_numpy(raw).cuda(), torch.from_numpy(sc.view(np.int16)).cuda(), deq)
    np.testing.assert_allclose(deq.cpu().numpy(), Wp, rtol=0, atol=1e-6 * np.abs(Wp).max())


@pytest.fixture(scope="module")
def c5_ref():
    w = wl("c5")
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    return w, Pl, Pr, Pr.rotate_rows(Pl.rotate_cols(synth.x_as_f64(w)))


@pytest.mark.parametrize("qi", [0, 1])
def test_c5_forward_full(c5_ref, qi):
    w, Pl, Pr, ref = c5_ref
    q = w.quants[qi]
    _full_forward(w, Pl, Pr, ref, q, f"c5 {q.kind} {q.bits}-bit")


@pytest.mark.parametrize("qi", [0, 1])
def test_c5_inverse_full(qi):
    w = wl("c5")
    q = w.quants[qi]
    Pl, Pr = oracle.processor(w.left), oracle.processor(w.right)
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    raw, sc = synth.random_code_stream(5050 + qi, w.rows, w.cols, q.bits, q.group)
    _inverse_full(w, left, right, q, raw, sc, Pl, Pr, f"c5 {q.kind} {q.bits}-bit random stream")


# ------------------------------------------------------------ small shapes, every radix path

RADICES = [(2, 4), (4, 4), (8, 2, 4), (3, 5), (7,), (16, 16), (5, 3, 2), (64, 4), (43, 2),
           (2, 2, 2, 2, 2, 2), (1, 8), (6, 6), (32, 16, 16)]


@pytest.mark.parametrize("radix", RADICES)
@pytest.mark.parametrize("side", ["right", "left"])
def test_small_rotate_both_directions(radix, side):
    d = int(np.prod(radix))
    s = synth.side_draws(700 + d, radix, "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    P = oracle.processor(s)
    plan = harp.Plan.from_side(s)
    nvec = 37                                  # ragged against every tile size
    if side == "right":
        X = synth.small_matrix(d, nvec, d)
        sd, rot = harp.HARP_RIGHT, P.rotate_rows
        buf_shape, view = (nvec, ((d + 3) // 4) * 4), (slice(None), slice(0, d))
    else:
        X = synth.small_matrix(d, d, nvec)
        sd, rot = harp.HARP_LEFT, P.rotate_cols
        buf_shape, view = (d, 40), (slice(None), slice(0, nvec))
    Xf = X.astype(np.float32).astype(np.float64)
    xb = torch.zeros(buf_shape, dtype=torch.float32, device="cuda")
    xv = xb[view]
    xv.copy_(torch.from_numpy(X.astype(np.float32)))
    ob = torch.full(buf_shape, 7.0, dtype=torch.float32, device="cuda")
    ov = ob[view]
    harp.harp_rotate(plan, sd, harp.HARP_FWD, xv, ov)
    assert rel_l2(ov.cpu().numpy(), rot(Xf)) <= TOL_F32
    # padding outside the view is untouched
    mask = torch.ones(buf_shape, dtype=torch.bool, device="cuda")
    mask[view] = False
    assert torch.all(ob[mask] == 7.0)
    harp.harp_rotate(plan, sd, harp.HARP_INV, xv, ov)
    assert rel_l2(ov.cpu().numpy(), rot(Xf, inverse=True)) <= TOL_F32
    # bf16 in, bf16 out (padded leading dimension)
    x16b = torch.zeros(buf_shape, dtype=torch.bfloat16, device="cuda")
    x16 = x16b[view]
    x16.copy_(xv)
    X16 = x16.float().cpu().numpy().astype(np.float64)
    o16b = torch.zeros(buf_shape, dtype=torch.bfloat16, device="cuda")
    o16 = o16b[view]
    harp.harp_rotate(plan, sd, harp.HARP_FWD, x16, o16)
    assert rel_l2(o16.float().cpu().numpy(), rot(X16)) <= TOL_BF16
    # bf16 in, fp32 out is exact-input fp32 arithmetic
    harp.harp_rotate(plan, sd, harp.HARP_FWD, x16, ov)
    assert rel_l2(ov.cpu().numpy(), rot(X16)) <= TOL_F32


@pytest.mark.parametrize("kind,bits,group", [("lloyd_max", 2, 32), ("lloyd_max", 3, 64),
                                             ("lloyd_max", 4, 128), ("absmax", 2, 64),
                                             ("absmax", 3, 512), ("absmax", 4, 32),
                                             ("lloyd_max", 5, 128), ("absmax", 5, 64)])
def test_standalone_quantize_and_dequantize(kind, bits, group):
    rows, cols = 33, 512
    X = synth.small_matrix(bits * 10 + group, rows, cols, outlier_cols=3, scale=0.02)
    X32 = X.astype(np.float32)
    oc, osc, m, sm = oracle.quantize(kind, bits, group, X32.astype(np.float64))
    cb = harp.Codebook(kind, bits, group)
    x = torch.from_numpy(X32).cuda()
    codes, scales = harp.empty_codes(rows, cols, cb)
    harp.harp_quantize(cb, x, codes, scales)
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
    deq = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    harp.harp_dequantize(cb, codes, scales, deq)
    gc = np_unpack(codes.cpu().numpy(), bits, cols)
    ref = oracle.dequantize(kind, bits, group, oc, osc)
    same = (gc == oc) & (scales_np(scales) == osc).repeat(group, axis=1)
    np.testing.assert_allclose(deq.cpu().numpy()[same], ref[same], rtol=1e-7, atol=0)


def test_edge_cases_zero_rows_huge_values_and_empty():
    cb = harp.Codebook("lloyd_max", 4, 128)
    X = np.zeros((3, 256), np.float32)
    X[1, :128] = 1e6            # RMS above the fp16 range: scale saturates at 65504
    X[2] = synth.small_matrix(3, 1, 256)[0]
    oc, osc, m, sm = oracle.quantize("lloyd_max", 4, 128, X.astype(np.float64))
    codes, scales = harp.empty_codes(3, 256, cb)
    harp.harp_quantize(cb, torch.from_numpy(X).cuda(), codes, scales)
    s = scales_np(scales)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0x7BFF
    compare_quant(codes.cpu().numpy(), s, oc, osc, m, sm, 4, 128)
    gc = np_unpack(codes.cpu().numpy(), 4, 256)
    assert np.all(gc[0] == 8)
    # empty matrices launch nothing and succeed
    s16 = synth.side_draws(1, (16, 16), "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan = harp.Plan.from_side(s16)
    e = torch.empty((0, 256), dtype=torch.float32, device="cuda")
    c0, sc0 = harp.empty_codes(0, 256, cb)
    harp.harp_rotate_quantize(None, plan, cb, e, c0, sc0)
    harp.harp_rotate(plan, harp.HARP_RIGHT, harp.HARP_FWD, e, torch.empty_like(e))
    torch.cuda.synchronize()


def test_plan_info_and_workspace():
    s = synth.side_draws(5, (43, 16, 16), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan = harp.Plan.from_side(s)
    assert plan.info() == (11008, 3, (43, 16, 16))
    assert harp.workspace_size(plan, plan, 11008, 11008) == 11008 * 11008 * 8
    assert harp.workspace_size(None, plan, 7, 11008) == 0


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs a second device to make the current one differ from the plan's")
def test_calls_refuse_a_plan_of_another_device():
    """A plan's blocks live on the device that was current at creation; every
    launching call made with another device current returns
    HARP_ERR_INVALID_ARG before touching memory."""
    torch.cuda.set_device(0)
    s16 = synth.side_draws(1, (16, 16), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    plan = harp.Plan.from_side(s16)
    cb = harp.Codebook("lloyd_max", 4, 128)
    try:
        torch.cuda.set_device(1)
        st = harp.lib().harp_rotate(plan.handle, harp.HARP_RIGHT, harp.HARP_FWD, None, harp.HARP_F32,
                                    None, harp.HARP_F32, 4, 256, 256, 256, None)
        assert st == 1
        st = harp.lib().harp_rotate_quantize(None, plan.handle, cb.handle, None, harp.HARP_F32, 4, 256,
                                             None, None, None, None, 0, None)
        assert st == 1
        st = harp.lib().harp_rotate_quantize_static(plan.handle, plan.handle, cb.handle, None,
                                                    harp.HARP_F32, 256, 256, None, None, None, None)
        assert st == 1
    finally:
        torch.cuda.set_device(0)


def test_pass_events_time_each_pass():
    """harp_pass_count reports the pass kernels of the two-sided calls and
    harp_set_pass_events gets one event per pass boundary recorded; results
    do not change when events are registered."""
    w = wl("c2")
    q = w.quants[0]
    left, right = harp.Plan.from_side(w.left), harp.Plan.from_side(w.right)
    cb = harp.Codebook(q.kind, q.bits, q.group)
    n = harp.harp_pass_count(left, right, cb)
    assert n >= 2
    assert harp.harp_pass_count(None, right, cb) == 0
    # every stage of both processors is applied by exactly one pass
    assert sum(harp.harp_pass_fma(left, right, cb, k) for k in range(n)) == 2 * 48
    x = to_dev(w)
    codes, scales, _ = harp.rotate_quantize(left, right, cb, x)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    harp.harp_set_pass_events(evs)
    try:
        codes2, scales2, _ = harp.rotate_quantize(left, right, cb, x)
    finally:
        harp.harp_set_pass_events([])
    torch.cuda.synchronize()
    times = [evs[k].elapsed_time(evs[k + 1]) for k in range(n)]
    assert all(t > 0 for t in times)
    assert torch.equal(codes2, codes) and torch.equal(scales2, scales)


def test_hadamard_two_sided_matches_oracle():
    """Hadamard-initialised processors on both sides (HARP section 2.2,
    theta = 0: random signs times normalised Sylvester blocks), which the
    pass kernels apply as Walsh-Hadamard butterflies: the forward rotation +
    4-bit Lloyd-Max, and the inverse of a random code stream, match the
    oracle."""
    left_s = synth.side_draws(21, (16, 8, 8), "hadamard", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(21, (16, 16, 8), "hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    rows, cols = 1024, 2048
    W = synth.small_matrix(22, rows, cols, outlier_cols=4, scale=0.02)
    Wb = synth.to_bf16_bits(W)
    Pl, Pr = oracle.processor(left_s), oracle.processor(right_s)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.bf16_bits_to_f64(Wb), Pl, Pr, "lloyd_max", 4, 128)
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    cb = harp.Codebook("lloyd_max", 4, 128)
    assert harp.harp_pass_count(left, right, cb) >= 2
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(left, right, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, 4, 128)
    raw, sc = synth.random_code_stream(23, rows, cols, 4, 128)
    ref3 = oracle.dequantize_unrotate(oracle.unpack(4, raw, cols), sc, Pl, Pr, "lloyd_max", 4, 128)
    out = harp.dequantize_unrotate(left, right, cb, torch.from_numpy(raw).cuda(),
                                   torch.from_numpy(sc.view(np.int16)).cuda(), rows, cols, torch.float32)
    assert rel_l2(out.cpu().numpy(), ref3) <= TOL_F32


def test_mixed_radix_5120_two_sided(block_stages):
    """HARP section 2.1's arbitrary-d example, 5120 = 8 * 8 * 8 * 5 * 2, as
    the column processor of a 5120 x 1280 weight (row processor (5, 16, 16)),
    random orthogonal blocks: the fused forward with 3-bit Lloyd-Max g128 and
    the inverse of its codes against the oracle, element by element."""
    left_s = synth.side_draws(31, (8, 8, 8, 5, 2), "qr", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(31, (5, 16, 16), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    rows, cols = 5120, 1280
    W = synth.small_matrix(32, rows, cols, outlier_cols=6, scale=0.02)
    Wb = synth.to_bf16_bits(W)
    Pl, Pr = oracle.processor(left_s), oracle.processor(right_s)
    ref, oc, _, osc, m, sm = oracle.rotate_quantize(synth.bf16_bits_to_f64(Wb), Pl, Pr, "lloyd_max", 3, 128)
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    cb = harp.Codebook("lloyd_max", 3, 128)
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, rot = harp.rotate_quantize(left, right, cb, xb, want_rotated=True)
    assert rel_l2(rot.cpu().numpy(), ref) <= TOL_F32
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, 3, 128)
    # the inverse of the oracle's own codes (no oracle input comes from the CUDA path)
    ref_inv = oracle.dequantize_unrotate(oc, osc, Pl, Pr, "lloyd_max", 3, 128)
    out = harp.dequantize_unrotate(left, right, cb, torch.from_numpy(oracle.pack(3, oc)).cuda(),
                                   torch.from_numpy(osc.view(np.int16)).cuda(), rows, cols, torch.float32)
    assert rel_l2(out.cpu().numpy(), ref_inv) <= TOL_F32



def test_no_kernel_wait_ran_out():
    """Every wait inside the library's kernels is bounded and records when it
    runs out; none did during the tests above."""
    assert harp.harp_fault_status() == 0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_absmax_scale_mode_every_kernel(bits):
    """The alternative Lloyd-Max scale s = max|x| / c_{K-1} (HARP_SCALE_ABSMAX)
    in every quantizer the library has, against the oracle in the same mode:
    the standalone codec, the two-sided pass kernels, the whole-vector kernel
    (right-only rows of 4096) and the short-vector kernel (rows of 128)."""
    group = 128
    cb = harp.Codebook("lloyd_max", bits, group, scale_mode="absmax")
    # standalone codec
    X = synth.small_matrix(40 + bits, 33, 512, outlier_cols=3, scale=0.02).astype(np.float32)
    oc, osc, m, sm = oracle.quantize("lloyd_max", bits, group, X.astype(np.float64), scale_mode="absmax")
    codes, scales = harp.empty_codes(33, 512, cb)
    harp.harp_quantize(cb, torch.from_numpy(X).cuda(), codes, scales)
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
    # two-sided pass kernels (1024 x 2048)
    left_s = synth.side_draws(41, (16, 8, 8), "qr", synth.S_SIGNS_L, synth.S_BLOCKS_L)
    right_s = synth.side_draws(41, (16, 16, 8), "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
    W = synth.small_matrix(42, 1024, 2048, outlier_cols=4, scale=0.02)
    Wb = synth.to_bf16_bits(W)
    Pl, Pr = oracle.processor(left_s), oracle.processor(right_s)
    ref = Pr.rotate_rows(Pl.rotate_cols(synth.bf16_bits_to_f64(Wb)))
    oc, osc, m, sm = oracle.quantize("lloyd_max", bits, group, ref, scale_mode="absmax")
    left, right = harp.Plan.from_side(left_s), harp.Plan.from_side(right_s)
    assert harp.harp_pass_count(left, right, cb) >= 2
    xb = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, _ = harp.rotate_quantize(left, right, cb, xb)
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
    # right-only rows: the row kernel (radices 8) and the whole-vector kernel (a radix 7)
    for radix in ((8, 8, 8, 8), (8, 8, 8, 7)):
        rs = synth.side_draws(43, radix, "qr", synth.S_SIGNS_R, synth.S_BLOCKS_R)
        d = int(np.prod(radix))
        Xr = synth.small_matrix(44, 40, d, outlier_cols=4).astype(np.float32)
        P = oracle.processor(rs)
        ref = P.rotate_rows(Xr.astype(np.float64))
        oc, osc, m, sm = oracle.quantize("lloyd_max", bits, group, ref, scale_mode="absmax")
        codes, scales, _ = harp.rotate_quantize(None, harp.Plan.from_side(rs), cb, torch.from_numpy(Xr).cuda())
        compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
    # short-vector kernel: rows of 128 (bf16 in)
    h128 = harp.Plan((16, 8), [harp.stage_blocks("hadamard", b, 128 // b) for b in (16, 8)])
    Ph = oracle.Processor((16, 8), [oracle.stage_blocks("hadamard", b, 128 // b) for b in (16, 8)])
    Xs = synth.to_bf16_bits(synth.small_matrix(45, 600, 128, outlier_cols=2, scale=0.02))
    ref = Ph.rotate_rows(synth.bf16_bits_to_f64(Xs))
    oc, osc, m, sm = oracle.quantize("lloyd_max", bits, group, ref, scale_mode="absmax")
    xs = torch.from_numpy(Xs.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales, _ = harp.rotate_quantize(None, h128, cb, xs)
    compare_quant(codes.cpu().numpy(), scales_np(scales), oc, osc, m, sm, bits, group)
