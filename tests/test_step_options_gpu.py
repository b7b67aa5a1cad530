"""GPU parity of the step's options against the fp64 oracle.

* update scale modes ('spectral', 'rms_norm') and extra_scale_factor: the
  weight change within 1e-5 relative of the oracle's, fed the same
  Newton-Schulz output;
* row sums of squares left by the Newton-Schulz call (row_sumsq) on every
  path (GEMM wide and tall, fused wide, fused tall, head views): within fp32
  summation error of the sums of the stored output, the output itself
  unchanged bit for bit, and NorMuon fed from them within 1e-5 of the oracle;
* Gram restarts: rank-deficient slices stay in the quintic's band
  (sigma_max <= 1.25, as the standard form), and the device is as close to
  the exact result as a numpy model of the same storage precisions.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from precision_model import ns_gram_f16

pytestmark = pytest.mark.gpu
DEV = "cuda"
NS_TOL = 3e-2


@pytest.fixture(scope="module")
def mn():
    import newton_schulz_ns_b200 as m
    return m


def f64(t):
    return t.detach().float().cpu().double().numpy()


def h32(x):
    return float(np.float32(x))


def rel(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def _aligned(n, r, c, dtype, fill=0.0):
    ld = (c + 7) // 8 * 8
    return torch.full((n, r, ld), fill, dtype=dtype, device=DEV)[:, :, :c]


def _seeded(n, r, c, seed, dtype, std=1.0):
    g = torch.Generator().manual_seed(seed)
    t = _aligned(n, r, c, dtype)
    t.copy_((torch.randn((n, r, c), generator=g) * std).to(dtype).to(DEV))
    return t


def _run(mn, batches, variant, hp):
    ws = mn.allocate_workspace(batches, 1 if variant == "standard" else 2)
    (mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched)(batches, hp, ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0


# ----------------------------------------------------------------- update scale modes

@pytest.mark.parametrize("mode", ["spectral", "rms_norm"])
@pytest.mark.parametrize("extra", [0.5, 1.0, 2.5])
@pytest.mark.parametrize("shape,fan", [((2, 300, 200), (300, 200)), ((4, 64, 576), (64, 576)),
                                       ((4, 128, 512), (512, 512))])     # last: head slices of a 512 x 512
def test_update_scale_modes_and_extra_factor(mn, mode, extra, shape, fan):
    n, r, c = shape
    O = _seeded(n, r, c, 70, torch.bfloat16, std=1 / math.sqrt(c))
    W = _seeded(n, r, c, 71, torch.float32, std=0.02)
    W0 = W.clone()
    V = torch.rand((n, r), generator=torch.Generator().manual_seed(72)).mul(1e-3).to(DEV)
    V0 = V.clone()
    b = mn.Batch(n, r, c, ns_out=O, weight=W, variance=V, fan_out=fan[0], fan_in=fan[1])
    hp = mn.Hparams(lr=0.02, weight_decay=0.01, scale_mode=mode, extra_scale_factor=extra)
    ws = mn.allocate_workspace([b], 3)
    mn.normuon_update([b], hp, True, ws)
    torch.cuda.synchronize()
    scale = oracle.update_scale(*fan, mode=mode, extra=h32(extra))
    ref = oracle.muon_step_slices(np.zeros((n, r, c)), np.zeros((n, r, c)), f64(W0), f64(V0), normuon=True,
                                  beta2=h32(0.95), nor_eps=h32(1e-8), lr=h32(0.02), weight_decay=h32(0.01),
                                  lr_scale=h32(scale), O_override=f64(O))
    dW = f64(W) - f64(W0)
    assert rel(dW, ref["W"] - f64(W0)) < 1e-5
    assert rel(f64(V), ref["v"]) < 1e-5


# ----------------------------------------------------------------- row sums from the Newton-Schulz call

ROW_CASES = [
    (3, 300, 520),     # GEMM path, wide
    (2, 520, 300),     # GEMM path, tall (iterated transposed, output rows = parameter rows)
    (1, 256, 256),     # GEMM path, square
    (3, 64, 576),      # fused, wide (conv megabatch slice)
    (2, 100, 1000),    # fused, wide, ragged column blocks
    (2, 576, 64),      # fused, tall (transposed copy)
    (2, 33, 45),       # fused, element stores
]


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", ROW_CASES)
def test_ns_leaves_row_sums_of_its_output(mn, variant, shape):
    n, r, c = shape
    U = _seeded(n, r, c, 80 + r + c, torch.bfloat16)
    plain = mn.Batch(n, r, c, ns_in=U, ns_out=_aligned(n, r, c, torch.bfloat16, float("nan")))
    _run(mn, [plain], variant, mn.Hparams())
    for fused in (1, 0):
        rs = torch.full((n * r,), float("nan"), device=DEV)
        b = mn.Batch(n, r, c, ns_in=U, ns_out=_aligned(n, r, c, torch.bfloat16, float("nan")), row_sumsq=rs)
        with mn.testing_options(fused_small=fused):
            _run(mn, [b], variant, mn.Hparams())
        O = f64(b.ns_out)
        want = np.sum(O * O, axis=2).reshape(-1)
        got = f64(rs)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want) / np.maximum(want, 1e-30)) < 1e-5, (fused, np.max(np.abs(got - want)))
        if fused:
            assert torch.equal(b.ns_out, plain.ns_out)            # asking for the sums changes nothing else


def test_row_sums_of_head_views(mn):
    H, d, c = 8, 64, 384
    W = _seeded(1, H * d, c, 90, torch.bfloat16)[0]
    heads = W.view(H, d, c) if W.is_contiguous() else W.reshape(H, d, c)
    rs = torch.full((H * d,), float("nan"), device=DEV)
    out = torch.empty_like(heads)
    b = mn.Batch(H, d, c, ns_in=heads, ns_out=out, row_sumsq=rs)
    _run(mn, [b], "standard", mn.Hparams())
    O = f64(out)
    want = np.sum(O * O, axis=2).reshape(-1)
    assert np.max(np.abs(f64(rs) - want) / want) < 1e-5


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_normuon_from_row_sums_matches_oracle_and_the_reading_pass(mn, variant):
    shapes = [(4, 64, 576), (2, 300, 520), (2, 520, 300), (2, 576, 64)]
    results = []
    for use_rs in (True, False):
        bs, before = [], []
        for k, (n, r, c) in enumerate(shapes):
            U = _seeded(n, r, c, 100 + k, torch.bfloat16)
            W = _seeded(n, r, c, 110 + k, torch.float32, std=0.02)
            V = torch.rand((n, r), generator=torch.Generator().manual_seed(120 + k)).mul(1e-3).to(DEV)
            before.append((f64(W), f64(V)))
            bs.append(mn.Batch(n, r, c, ns_in=U, ns_out=_aligned(n, r, c, torch.bfloat16), weight=W,
                               variance=V.reshape(-1), fan_out=r, fan_in=c,
                               row_sumsq=torch.zeros(n * r, device=DEV) if use_rs else None))
        hp = mn.Hparams(lr=0.02, weight_decay=0.01)
        ws = mn.allocate_workspace(bs, -1)
        (mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched)(bs, hp, ws)
        mn.normuon_update(bs, hp, True, ws)
        torch.cuda.synchronize()
        assert mn.workspace_error(ws) == 0
        for b, (W0, V0) in zip(bs, before):
            ref = oracle.muon_step_slices(np.zeros(W0.shape), np.zeros(W0.shape), W0, V0, normuon=True,
                                          beta2=h32(0.95), nor_eps=h32(1e-8), lr=h32(0.02),
                                          weight_decay=h32(0.01), lr_scale=h32(oracle.update_scale(b.rows, b.cols)),
                                          O_override=f64(b.ns_out))
            assert rel(f64(b.variance).reshape(V0.shape), ref["v"]) < 1e-5
            assert rel(f64(b.weight) - W0, ref["W"] - W0) < 1e-5
        results.append([(f64(b.ns_out), f64(b.weight)) for b in bs])
    for (o1, w1), (o2, w2) in zip(*results):
        assert np.array_equal(o1, o2)
        assert np.max(np.abs(w1 - w2)) <= 1e-6 * np.max(np.abs(w2))


# ----------------------------------------------------------------- Gram restarts

def _low_rank(n, r, c, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(n, r, k, generator=g) @ torch.randn(n, k, c, generator=g)).to(torch.bfloat16)
    t = _aligned(n, r, c, torch.bfloat16)
    t.copy_(x.to(DEV))
    return t


@pytest.mark.parametrize("shape,rank", [((100, 160), 3), ((640, 100), 3), ((300, 520), 5), ((520, 300), 5),
                                        ((128, 4096), 4), ((100, 350), 1), ((256, 896), 1), ((896, 256), 1),
                                        ((512, 1792), 1)])
def test_gram_rank_deficient_stays_in_band(mn, shape, rank):
    # Without restarts, fp16 rounding gives A = X X^T small negative
    # eigenvalues in its null space, which A <- P A P grows by about a^2 per
    # step; a float32 model of the storage precisions puts the top singular
    # value of rank-1 inputs at 2.4 (m = 100), 1.7 (256), 1.4 (512), 1.26
    # (1024) and 1.14 (2048), of rank-3 ones at up to 1.6 (m = 100).
    r, c = shape
    U = _low_rank(3, r, c, rank, 130 + r)
    b = mn.Batch(3, r, c, ns_in=U, ns_out=_aligned(3, r, c, torch.bfloat16, float("nan")))
    _run(mn, [b], "gram", mn.Hparams())
    x, got = f64(U), f64(b.ns_out)
    ref = oracle.ns_batched(x, "gram", restart=3)
    for i in range(3):
        assert np.all(np.isfinite(got[i]))
        smax = float(np.linalg.norm(got[i], 2))
        assert smax <= 1.25, (shape, i, smax)
        # as close to the exact result as the storage precisions allow
        model = ns_gram_f16(x[i], restart=3)
        assert rel(got[i], ref[i]) <= max(3 * rel(model, ref[i]), NS_TOL), (rel(got[i], ref[i]), rel(model, ref[i]))


@pytest.mark.parametrize("restart", [0, 1, 2, 3])
@pytest.mark.parametrize("shape,steps", [((128, 1024), 5), ((300, 200), 5), ((256, 768), 7), ((96, 700), 16),
                                         ((128, 4096), 5), ((96, 6000), 7)])
def test_gram_restart_periods_match_oracle(mn, restart, shape, steps):
    r, c = shape
    U = _seeded(2, r, c, 140 + r, torch.bfloat16)
    b = mn.Batch(2, r, c, ns_in=U, ns_out=_aligned(2, r, c, torch.bfloat16, float("nan")))
    _run(mn, [b], "gram", mn.Hparams(ns_steps=steps, gram_restart=restart))
    ref = oracle.ns_batched(f64(U), "gram", steps=steps, restart=restart)
    for i in range(2):
        assert rel(f64(b.ns_out)[i], ref[i]) < NS_TOL, (restart, shape, steps, rel(f64(b.ns_out)[i], ref[i]))
