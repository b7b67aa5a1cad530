"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formulas: each checks it against a
closed form (the singular-value form of an odd matrix polynomial, geometric
series), an invariant (orthogonal equivariance, transpose, zero padding,
norm preservation), a special case that reduces to a library routine, or a
value the pages print (golden fixtures under tests/golden/, each with its
citation).
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
import oracle as orc

ABC = (3.4445, -4.7750, 2.0315)       # the quintic coefficients as the pages list them


def _p5(s, steps=5):
    """Scalar quintic p(s) = a s + b s^3 + c s^5 applied ``steps`` times."""
    a, b, c = ABC
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def _svd_form(X, eps=1e-7, steps=5):
    """Newton-Schulz of X in closed form: an odd polynomial acts on singular values."""
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    nrm = math.sqrt(float(np.sum(X * X))) + eps
    return (U * _p5(S / nrm, steps)) @ Vt


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


SHAPES = [(1, 1), (1, 7), (7, 1), (3, 5), (64, 576), (200, 300), (300, 200), (256, 256), (130, 17)]


# ------------------------------------------------------------- Newton-Schulz

@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_ns_matches_singular_value_closed_form(shape, variant):
    rng = np.random.default_rng(hash(shape) % 2**31)
    X = rng.standard_normal(shape) * 3.0
    fn = orc.newton_schulz if variant == "standard" else orc.gram_newton_schulz
    got = fn(X)
    assert got.shape == X.shape
    assert _rel(got, _svd_form(X)) < 1e-11


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_ns_eps_placement_small_norm(variant):
    # At ||X||_F ~ 1e-5 the +eps in the denominator moves singular values by 1e-2
    # relative, so a max(||X||, eps) or eps-free normalization fails this.
    rng = np.random.default_rng(7)
    X = rng.standard_normal((12, 20))
    X *= 1e-5 / np.linalg.norm(X)
    fn = orc.newton_schulz if variant == "standard" else orc.gram_newton_schulz
    assert _rel(fn(X), _svd_form(X)) < 1e-11
    assert _rel(fn(X), _svd_form(X, eps=0.0)) > 1e-4


def test_ns_diagonal_input_iterates_scalar_polynomial():
    # A diagonal input stays diagonal and each entry follows p(s) on d_i/||d||.
    d = np.array([3.0, -1.0, 0.5, 0.0, 2.0])
    X = np.diag(d)
    got = orc.newton_schulz(X)
    want = np.diag(_p5(d / (np.linalg.norm(d) + 1e-7)))
    assert np.max(np.abs(got - want)) < 1e-13


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_ns_orthogonal_equivariance_and_transpose(variant):
    rng = np.random.default_rng(11)
    X = rng.standard_normal((24, 40))
    P, _ = np.linalg.qr(rng.standard_normal((24, 24)))
    R, _ = np.linalg.qr(rng.standard_normal((40, 40)))
    fn = orc.newton_schulz if variant == "standard" else orc.gram_newton_schulz
    base = fn(X)
    assert _rel(fn(P @ X @ R.T), P @ base @ R.T) < 1e-12
    assert _rel(fn(X.T), base.T) < 1e-12


@pytest.mark.parametrize("shape", [(256, 256), (64, 576), (128, 4096), (512, 1024), (1024, 512)])
def test_gram_equals_standard(shape):
    rng = np.random.default_rng(3)
    X = rng.standard_normal(shape)
    assert _rel(orc.gram_newton_schulz(X), orc.newton_schulz(X)) < 1e-10


def test_ns_converges_towards_orthogonal():
    # Singular values land in the band the quintic maps [0,1] into after 5 steps.
    rng = np.random.default_rng(5)
    X = rng.standard_normal((64, 256))
    s = np.linalg.svd(orc.newton_schulz(X), compute_uv=False)
    assert s.min() > 0.6 and s.max() < 1.25


def test_megabatch_equals_separate_calls_bitwise():
    rng = np.random.default_rng(1)
    U = rng.standard_normal((5, 8, 36))
    batched = orc.ns_batched(U)
    for i in range(5):
        assert np.array_equal(batched[i], orc.newton_schulz(U[i]))
    rev = orc.ns_batched(U[::-1].copy())
    assert np.array_equal(rev[::-1], batched)


@pytest.mark.parametrize("row", read_golden("per_head_identity.txt"))
def test_per_head_shard_equals_block_of_whole(row):
    r, c, heads, tp = (int(v) for v in row[:4])
    variant, printed = row[4], float(row[5])
    rng = np.random.default_rng(2)
    W = rng.standard_normal((r, c))
    whole = orc.per_head_ns(W, heads, variant)
    rows_per = r // tp
    for k in range(tp):
        shard = orc.per_head_ns(W[k * rows_per:(k + 1) * rows_per], heads // tp, variant)
        diff = float(np.max(np.abs(shard - whole[k * rows_per:(k + 1) * rows_per])))
        assert diff == printed


@pytest.mark.parametrize("row", read_golden("shard_vs_whole.txt"))
def test_row_shard_differs_from_rows_of_whole(row):
    shape = tuple(int(v) for v in row[0].split("x"))
    variant, tp, split, block = row[1], int(row[2]), row[3], row[4]
    printed, tol = float(row[5]), float(row[6])
    fn = orc.newton_schulz if variant == "standard" else orc.gram_newton_schulz
    rng = np.random.default_rng(0)
    G = rng.standard_normal(shape)
    whole = fn(G)
    axis = 0 if split == "dim0" else 1
    parts = np.split(G, tp, axis=axis)
    wparts = np.split(whole, tp, axis=axis)
    if block == "all":
        got = _rel(np.concatenate([fn(p) for p in parts], axis=axis), whole)
    else:
        k = int(block)
        got = _rel(fn(parts[k]), wparts[k])
    assert abs(got - printed) <= tol, (got, printed)


def test_zero_padding_leaves_real_columns_unchanged():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((20, 30))
    Xp = np.concatenate([X, np.zeros((20, 9))], axis=1)
    got = orc.newton_schulz(Xp)
    assert np.all(got[:, 30:] == 0.0)
    assert np.max(np.abs(got[:, :30] - orc.newton_schulz(X))) < 1e-14
    Xr = np.concatenate([X, np.zeros((5, 30))], axis=0)
    gotr = orc.newton_schulz(Xr)
    assert np.all(gotr[20:] == 0.0)
    assert np.max(np.abs(gotr[:20] - orc.newton_schulz(X))) < 1e-14


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_zero_and_rank_deficient_inputs(variant):
    fn = orc.newton_schulz if variant == "standard" else orc.gram_newton_schulz
    assert np.all(fn(np.zeros((6, 9))) == 0.0)
    rng = np.random.default_rng(9)
    X = rng.standard_normal((10, 3)) @ rng.standard_normal((3, 16))      # rank 3
    s = np.linalg.svd(fn(X), compute_uv=False)
    assert np.sum(s > 1e-8) == 3
    assert _rel(fn(X), _svd_form(X)) < 1e-10


def _conv_rows():
    return read_golden("conv_flatten.txt")


@pytest.mark.parametrize("row", _conv_rows())
def test_conv_megabatch_steps_like_flattened_matrices(row):
    stacked = tuple(int(v) for v in row[1].split(","))
    flat = tuple(int(v) for v in row[2].split(","))
    rng = np.random.default_rng(6)
    Gs = rng.standard_normal(stacked)
    Ws = rng.standard_normal(stacked) * 0.02
    Mz = np.zeros(flat)
    v0 = np.zeros(flat[:2])
    Gf = orc.flatten_megabatch(Gs)
    assert Gf.shape == flat
    kw = dict(normuon=True, lr=0.02, weight_decay=0.01, lr_scale=orc.spectral_scale(flat[1], flat[2]))
    batched = orc.muon_step_slices(Gf, Mz, orc.flatten_megabatch(Ws), v0, **kw)
    for i in range(flat[0]):
        one = orc.muon_step_slices(Gs[i].reshape(1, flat[1], -1), Mz[:1], Ws[i].reshape(1, flat[1], -1),
                                   v0[:1], **kw)
        assert np.array_equal(one["W"][0], batched["W"][i])
        assert np.array_equal(one["v"][0], batched["v"][i])
    if row[3] != "-":
        # Negative control: orthogonalizing across the stack ([N, numel]) is a different map.
        wrong = tuple(int(v) for v in row[3].split(","))
        U = batched["U"].reshape(wrong)
        o_wrong = orc.newton_schulz(U).reshape(flat)
        assert _rel(o_wrong, batched["O"]) > 0.1


# ------------------------------------------------------------- momentum

def test_momentum_geometric_closed_form():
    rng = np.random.default_rng(8)
    G = rng.standard_normal((4, 6))
    mu = 0.95
    M = np.zeros_like(G)
    for k in range(1, 6):
        M, U = orc.momentum_nesterov(G, M, mu, nesterov=True)
        geo = (1 - mu ** k) / (1 - mu)
        assert np.allclose(M, geo * G, rtol=1e-14, atol=0)
        assert np.allclose(U, (1 + mu * geo) * G, rtol=1e-14, atol=0)
    M2, U2 = orc.momentum_nesterov(G, np.zeros_like(G), mu, nesterov=False)
    assert np.array_equal(U2, M2)


def test_ema_momentum_form_gives_same_orthogonal_input():
    # From zero, the EMA form (1-mu)G blend is (1-mu) times the sum form, so the
    # normalized Newton-Schulz input, and its output, agree.
    rng = np.random.default_rng(10)
    mu = 0.95
    M = np.zeros((16, 24))
    Me = np.zeros((16, 24))
    for _ in range(3):
        G = rng.standard_normal((16, 24))
        M, U = orc.momentum_nesterov(G, M, mu)
        Me = mu * Me + (1 - mu) * G
        Ue = (1 - mu) * G + mu * Me
        assert _rel(orc.newton_schulz(Ue), orc.newton_schulz(U)) < 1e-6


# ------------------------------------------------------------- NorMuon

def test_normuon_preserves_frobenius_norm():
    rng = np.random.default_rng(12)
    O = rng.standard_normal((32, 48)) * np.linspace(0.1, 3, 32)[:, None]
    v = np.abs(rng.standard_normal(32)) * 0.1
    Oh, _ = orc.normuon_normalize(O, v, 0.95, 1e-8)
    assert abs(np.linalg.norm(Oh) / np.linalg.norm(O) - 1) < 1e-14


def test_normuon_identity_on_equal_row_rms():
    rng = np.random.default_rng(13)
    O = rng.standard_normal((16, 40))
    O /= np.sqrt(np.mean(O * O, axis=1, keepdims=True))           # every row RMS 1
    Oh, v = orc.normuon_normalize(O, np.zeros(16), 0.95, 1e-8)
    assert np.max(np.abs(Oh - O)) < 1e-13
    assert np.allclose(v, 0.05, rtol=1e-13)


def test_normuon_first_step_equalizes_row_rms():
    rng = np.random.default_rng(14)
    O = rng.standard_normal((10, 30)) * np.geomspace(1e-2, 10, 10)[:, None]
    Oh, _ = orc.normuon_normalize(O, np.zeros(10), 0.95, 0.0)
    rms = np.sqrt(np.mean(Oh * Oh, axis=1))
    assert np.max(rms) / np.min(rms) - 1 < 1e-12


def test_normuon_variance_geometric_closed_form():
    rng = np.random.default_rng(15)
    O = rng.standard_normal((5, 9))
    ms = np.array([sum(x * x for x in row) / 9 for row in O.tolist()])   # scalar loop
    v = np.zeros(5)
    for k in range(1, 5):
        _, v = orc.normuon_normalize(O, v, 0.9, 1e-8)
        assert np.allclose(v, (1 - 0.9 ** k) * ms, rtol=1e-13)


def test_normuon_zero_input_stays_zero():
    Oh, v = orc.normuon_normalize(np.zeros((3, 4)), np.zeros(3), 0.95, 1e-8)
    assert np.all(Oh == 0) and np.all(v == 0)


# ------------------------------------------------------------- update

@pytest.mark.parametrize("shape,scale", [((256, 256), 1.0), ((512, 1024), 1.0), ((1024, 512), math.sqrt(2.0)),
                                         ((14336, 4096), math.sqrt(3.5)), ((7168, 2048), math.sqrt(3.5)),
                                         ((64, 576), 1.0)])
def test_spectral_scale_values(shape, scale):
    assert orc.spectral_scale(*shape) == pytest.approx(scale, rel=1e-15)


def _orthogonal(r, c, seed):
    """An exactly orthogonal r x c matrix: orthonormal rows (r <= c) or columns (r > c)."""
    rng = np.random.default_rng(seed)
    q, _ = np.linalg.qr(rng.standard_normal((max(r, c), min(r, c))))
    return q.T if r <= c else q


@pytest.mark.parametrize("shape", [(64, 576), (576, 64), (256, 256), (128, 4096), (1024, 512), (1, 7)])
@pytest.mark.parametrize("extra", [1.0, 0.5])
def test_rms_norm_scale_gives_orthogonal_updates_rms_two_tenths(shape, extra):
    # The rms_norm mode's defining property: an orthogonalized update scaled
    # by it has element RMS 0.2 (times extra) whatever the shape.
    O = _orthogonal(*shape, seed=shape[0] + shape[1])
    U = orc.rms_norm_scale(*shape, extra) * O
    assert math.sqrt(float(np.mean(U * U))) == pytest.approx(0.2 * extra, rel=1e-12)
    assert orc.update_scale(*shape, mode="rms_norm", extra=extra) == orc.rms_norm_scale(*shape, extra)


@pytest.mark.parametrize("shape", [(576, 64), (256, 256), (1024, 512), (3584, 1024), (7, 1)])
def test_spectral_scale_gives_unit_rms_operator_norm_when_fan_out_ge_fan_in(shape):
    # ||s O||_{RMS->RMS} = sqrt(fan_in / fan_out) * ||s O||_2 = 1 for an orthogonal O.
    r, c = shape
    O = _orthogonal(r, c, seed=r + 2 * c)
    s = orc.update_scale(r, c, mode="spectral")
    assert math.sqrt(c / r) * s * np.linalg.norm(O, 2) == pytest.approx(1.0, rel=1e-12)


def test_update_scale_rejects_unknown_modes_and_empty_shapes():
    with pytest.raises(ValueError):
        orc.update_scale(4, 4, mode="shape")
    with pytest.raises(ValueError):
        orc.update_scale(0, 4)


def test_weight_update_closed_forms():
    rng = np.random.default_rng(16)
    Oh = rng.standard_normal((4, 5))
    W = rng.standard_normal((4, 5))
    assert np.allclose(orc.weight_update(np.zeros((4, 5)), Oh, 0.02, 0.01, 2.0), -0.04 * Oh, rtol=1e-15)
    assert np.allclose(orc.weight_update(W, np.zeros((4, 5)), 0.02, 0.01, 2.0), W * (1 - 2e-4), rtol=1e-15)


def test_bf16_round_matches_torch_and_ties_to_even():
    one = 1.0
    assert orc.bf16_round(one + 2.0 ** -8) == 1.0                 # tie -> even
    assert orc.bf16_round(one + 3 * 2.0 ** -8) == one + 2.0 ** -6  # tie -> even (up)
    rng = np.random.default_rng(17)
    x = rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(orc.bf16_round(x), want)


def test_full_step_storage_rounding():
    rng = np.random.default_rng(18)
    G = orc.bf16_round(rng.standard_normal((2, 8, 12)))
    M = np.zeros_like(G)
    W = orc.bf16_round(rng.standard_normal((2, 8, 12)) * 0.02)
    out = orc.muon_step_slices(G, M, W, np.zeros((2, 8)), normuon=True, mom_store="bf16", w_store="bf16")
    assert np.array_equal(out["M"], orc.bf16_round(out["M"]))
    assert np.array_equal(out["W"], orc.bf16_round(out["W"]))


def test_ns_flops_closed_forms():
    m = 512
    full = orc.ns_flops(m, m, "standard", triangle=False)
    tri = orc.ns_flops(m, m, "standard", triangle=True)
    assert full == 30 * m ** 3 and tri == 20 * m ** 3          # one triangle: a third off, square case
    assert orc.ns_flops(256, 1024, "gram") == 256 ** 2 * 1024 * 3 + 17 * 256 ** 3
    # one restart (before step 3 of 5): Q X and X X^T again; no P Q at step 3, no P A P at step 2
    assert orc.ns_flops(256, 1024, "gram", restart=3) == 256 ** 2 * 1024 * 6 + 14 * 256 ** 3


@pytest.mark.parametrize("shape", [(64, 576), (300, 200), (128, 128), (5, 3)])
@pytest.mark.parametrize("restart,steps", [(1, 5), (2, 5), (3, 5), (3, 16), (4, 16)])
def test_gram_with_restarts_equals_standard(shape, restart, steps):
    # A restart re-forms X = Q X and A = X X^T and resets Q: in exact
    # arithmetic nothing changes, with any per-step schedule.
    rng = np.random.default_rng(shape[0] * 7 + restart)
    U = rng.standard_normal(shape)
    sched = [(3.4445 - 0.03 * k, -4.7750 + 0.05 * k, 2.0315 - 0.02 * k) for k in range(steps)]
    ref = orc.newton_schulz(U, steps=steps, abc=sched)
    got = orc.gram_newton_schulz(U, steps=steps, abc=sched, restart=restart)
    assert np.max(np.abs(got - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref)))
    assert np.array_equal(orc.ns_batched(U[None], "gram", steps, abc=sched, restart=restart)[0], got)


# ----------------------------------------------------------------- Polar Express schedule (LP oracle)
# The minimax odd quintic for 1 on [lo, hi] is characterized by Chebyshev's
# alternation theorem: with three free coefficients, the error 1 - p
# attains its maximum modulus E at four points of alternating sign.  These
# pins check that property directly, the limit quintic near x = 1, and the
# interval recursion of the greedy schedule.

def _quintic(coef, x):
    return coef[0] * x + coef[1] * x ** 3 + coef[2] * x ** 5


@pytest.mark.parametrize("lo,hi", [(1e-3, 1.0), (0.1, 1.0), (0.5, 1.2), (0.02, 1.05)])
def test_polar_express_lp_equioscillates(lo, hi):
    coef, E = orc.minimax_quintic_lp(lo, hi)
    x = np.linspace(lo, hi, 400001)
    e = 1.0 - _quintic(coef, x)
    assert abs(np.abs(e).max() - E) <= 1e-5 * E
    # local extrema of e, with the endpoints
    d = np.diff(e)
    ext = [0] + [i + 1 for i in range(len(d) - 1) if d[i] * d[i + 1] < 0] + [len(x) - 1]
    vals = e[ext]
    big = vals[np.abs(vals) >= E * (1 - 1e-4)]
    assert len(big) >= 4
    signs = np.sign(big)
    assert np.all(signs[1:] != signs[:-1])      # alternating


def test_polar_express_lp_narrow_interval_tends_to_fixed_point_quintic():
    coef, E = orc.minimax_quintic_lp(0.99, 1.01)
    assert np.allclose(coef, orc.FIXED_POINT_QUINTIC, atol=3e-4)
    # p(1) = 1, p'(1) = p''(1) = 0 for the limit quintic
    a, b, c = orc.FIXED_POINT_QUINTIC
    assert a + b + c == 1.0 and a + 3 * b + 5 * c == 0.0 and 6 * b + 20 * c == 0.0


def test_polar_express_lp_schedule_recursion():
    coeffs, errs = orc.polar_express_lp(1e-3, 6)
    lo, hi = 1e-3, 1.0
    for coef, E in zip(coeffs, errs):
        mn, mx = orc.quintic_image(coef, lo, hi)
        # equioscillation: the image of the interval is [1 - E, 1 + E]
        assert abs(mn - (1 - E)) < 1e-5 and abs(mx - (1 + E)) < 1e-5
        lo, hi = mn, mx
    assert all(e2 < e1 for e1, e2 in zip(errs, errs[1:]))
    assert errs[-1] < 1e-3


def test_polar_express_lp_safety_scales_the_argument():
    s = 1.05
    (c1,), _ = orc.polar_express_lp(1e-2, 1, safety=1.0)
    (c2,), _ = orc.polar_express_lp(1e-2, 1, safety=s)
    assert np.allclose(c2, (c1[0] / s, c1[1] / s ** 3, c1[2] / s ** 5), rtol=1e-12)


def test_polar_express_schedule_drives_singular_values_into_the_band():
    # NS with a per-step schedule maps each normalized singular value through
    # the composed polynomials (odd polynomials act on singular values), so
    # a matrix whose normalized spectrum lies in [lower, 1] comes out inside
    # [1 - E_T, 1 + E_T].
    rng = np.random.default_rng(41)
    m, n = 24, 40
    Uo, _ = np.linalg.qr(rng.standard_normal((m, m)))
    Vo, _ = np.linalg.qr(rng.standard_normal((n, m)))
    sig = np.geomspace(1.0, 0.05, m)
    X = (Uo * sig) @ Vo.T
    lower = sig[-1] / np.linalg.norm(X) * 0.999
    coeffs, errs = orc.polar_express_lp(lower, 6)
    O = orc.newton_schulz(X, steps=6, eps=0.0, abc=coeffs)
    s_out = np.linalg.svd(O, compute_uv=False)
    assert np.all(np.abs(s_out - 1.0) <= errs[-1] * (1 + 1e-6) + 1e-12)
