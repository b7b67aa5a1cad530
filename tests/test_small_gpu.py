"""Parity of the fused small-side Newton-Schulz kernel with the fp64 oracle.

Slices with rows <= cols and rows <= 128 (the per-head [32, 128, 4096]
batch, the conv megabatch [16, 64, 576]) run the whole iteration in one
clustered launch and the cluster sums X X^T over distributed shared memory.
Up to 2048 columns each CTA keeps its column block of X resident in shared
memory; longer slices (columns a multiple of 8, up to 16384) stream their
column blocks through 4-CTA clusters from L2 at every step; the remaining
ones up to 4096 columns stay resident on 8 CTAs.  Both forms: the standard
one exchanges X X^T at every step; the Gram one exchanges X0 X0^T once (and
at each restart) and iterates on the m x m side in every CTA.  Tall slices
(rows > cols, cols <= 128) take the same kernels on a transposed copy.  The
shapes below cover every cluster split the planner picks (1 to 8 resident
CTAs of 64 to 512 columns, 4 streaming CTAs of 768 to 4096 columns), ragged
last blocks, CTAs that hold only padding, and short sides from 1 to 128.
Bars: 3e-2 relative Frobenius error against the oracle per slice (the
standard form iterates in fp16 here: 1e-2 where it is compared with the
GEMM path); bitwise batch invariance and run-to-run determinism; nothing
written outside the slice.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
NS_TOL = 3e-2


@pytest.fixture(scope="module")
def mn():
    import newton_schulz_ns_b200 as m
    return m


def f64(t):
    return t.detach().float().cpu().double().numpy()


def rel(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def _padded(n, r, c, dtype, fill, pad=8):
    ld = (c + 7) // 8 * 8 + pad
    base = torch.full((n, r, ld), fill, dtype=dtype, device=DEV)
    return base, base[:, :, :c]


def _seeded(n, r, c, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((n, r, c), generator=g) * std).to(torch.bfloat16)
    _, t = _padded(n, r, c, torch.bfloat16, 0.0)
    t.copy_(x.to(DEV))
    return t


def _ns(mn, U, hp=None, fused=True, variant="standard"):
    n, r, c = U.shape
    base, out = _padded(n, r, c, torch.bfloat16, float("nan"))
    b = mn.Batch(n, r, c, ns_in=U, ns_out=out)
    ws = mn.allocate_workspace([b], 1 if variant == "standard" else 2)
    fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    with mn.testing_options(fused_small=int(fused)):
        before = mn.kernel_launches()
        fn([b], hp or mn.Hparams(), ws)
        launches = mn.kernel_launches() - before
        torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    return base, out, launches


# (rows, cols): cluster split (CTAs x columns each) the planner picks.
# Columns resident in shared memory when they fit on 4 CTAs (cols <= 2048);
# longer slices (cols a multiple of 8, up to 16384) stream their columns
# through 4-CTA clusters in 64-column blocks; the rest up to 4096 columns
# stay resident on 8 CTAs.
SHAPES = [
    (64, 576),     # conv megabatch slice: resident 4 x 192, the last CTA partly padding
    (128, 4096),   # attention head: streamed 4 x 1024 (16 blocks per CTA)
    (128, 2000),   # resident 4 x 512, ragged last block
    (100, 1000),   # resident 4 x 256, ragged
    (128, 128),    # resident 2 x 64
    (3, 5),        # resident 1 x 64, element stores (cols not a multiple of 8)
    (64, 64),      # resident 1 x 64: a cluster of one, its partial X X^T is A
    (1, 4096),     # streamed; one row: one owner, three CTAs own no block of A
    (128, 4040),   # streamed 4 x 1024, last CTA's last blocks partly padding
    (65, 3000),    # streamed 4 x 768, 9 row blocks of A
    (33, 200),     # resident 4 x 64, 10 rows of A per CTA, one CTA only padding
    (50, 1001),    # resident 4 x 256, 14 rows of A per CTA, element stores
    (50, 4001),    # resident 8 x 512 (cols not a multiple of 8: not streamed)
    (128, 8192),   # streamed 4 x 2048 (past the resident limit)
    (96, 16384),   # streamed 4 x 4096, the longest fused slice
    (17, 5000),    # streamed 4 x 1280, ragged
    # tall slices: transposed into the workspace, fused, transposed back
    (576, 64),     # a channel-expanding conv slice
    (4096, 128),   # streamed on the transposed copy
    (1000, 100),
    (5, 3),
    (64, 40),      # a cluster of one on the transposed copy
    (3001, 65),    # resident 8 x 384, element stores on the transposed copy
    (12288, 80),   # streamed on the transposed copy
]


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", SHAPES)
def test_fused_small_matches_oracle(mn, shape, variant):
    r, c = shape
    U = _seeded(3, r, c, 500 + r + c)
    base, out, launches = _ns(mn, U, variant=variant)
    # error-word clear (1) + norms (2) + one fused launch (+ 2 transposes)
    assert launches <= (6 if r > c else 4)
    ref = oracle.ns_batched(f64(U), variant)
    got = f64(out)
    for i in range(3):
        assert rel(got[i], ref[i]) < NS_TOL, (shape, i, rel(got[i], ref[i]))
    # Nothing outside the slice was written.
    pad = base[:, :, c:]
    assert torch.isnan(pad.float()).all()


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("shape", [(64, 576), (128, 4096), (100, 1000)])
def test_fused_small_agrees_with_gemm_path(mn, shape, variant):
    r, c = shape
    U = _seeded(2, r, c, 900 + r)
    _, fused, nf = _ns(mn, U, fused=True, variant=variant)
    _, gemm, ng = _ns(mn, U, fused=False, variant=variant)
    assert nf < ng
    ref = oracle.ns_batched(f64(U), variant)
    for i in range(2):
        assert rel(f64(gemm)[i], ref[i]) < NS_TOL
        if variant == "standard":
            # fp16 iterates on the fused path (bf16 on the GEMM path): well inside the bar
            assert rel(f64(fused)[i], ref[i]) < 1e-2
        else:
            # the same arithmetic up to the order of fp32 sums
            assert rel(f64(fused)[i], ref[i]) < NS_TOL
            assert rel(f64(fused)[i], f64(gemm)[i]) < 1e-2


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_fused_small_batch_invariance_and_determinism(mn, variant):
    U = _seeded(40, 128, 1024, 77)
    _, all_out, _ = _ns(mn, U, variant=variant)
    _, again, _ = _ns(mn, U, variant=variant)
    assert torch.equal(all_out, again)
    for i in (0, 17, 39):
        _, one, _ = _ns(mn, U[i:i + 1].clone(), variant=variant)
        assert torch.equal(one[0], all_out[i])
    rev = U.flip(0).contiguous()
    _, rout, _ = _ns(mn, rev, variant=variant)
    assert torch.equal(rout.flip(0), all_out)


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_fused_small_many_slices(mn, variant):
    # Many more clusters than fit on the device at once: 300 slices of 8 CTAs.
    U = _seeded(300, 128, 4096, 31)
    _, out, launches = _ns(mn, U, variant=variant)
    assert launches <= 4
    ref = oracle.ns_batched(f64(U[::37]), variant)
    got = f64(out[::37])
    for i in range(ref.shape[0]):
        assert rel(got[i], ref[i]) < NS_TOL


@pytest.mark.parametrize("variant", ["standard", "gram"])
@pytest.mark.parametrize("steps", [1, 2, 3, 16])
def test_fused_small_steps_and_schedule(mn, steps, variant):
    sched = [(3.4445 - 0.05 * k, -4.7750 + 0.1 * k, 2.0315 - 0.05 * k) for k in range(steps)]
    U = _seeded(2, 96, 700, 8)
    _, out, _ = _ns(mn, U, mn.Hparams(ns_steps=steps, abc_schedule=sched), variant=variant)
    ref = oracle.ns_batched(f64(U), variant, steps=steps, abc=sched, restart=3 if variant == "gram" else 0)
    for i in range(2):
        assert rel(f64(out)[i], ref[i]) < NS_TOL


def test_fused_small_head_view_of_projection(mn):
    # q_proj 4096 x 4096 viewed as 32 heads of 128 rows: no copy, the batch
    # stride is 128 rows of the projection.
    g = torch.Generator().manual_seed(3)
    W = torch.randn((4096, 4096), generator=g).to(torch.bfloat16).to(DEV)
    heads = W.view(32, 128, 4096)
    out = torch.empty_like(heads)
    b = mn.Batch(32, 128, 4096, ns_in=heads, ns_out=out)
    ws = mn.allocate_workspace([b], 1)
    mn.muon_ns_batched([b], mn.Hparams(), ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    ref = oracle.per_head_ns(f64(W), 32, "standard")
    got = f64(out.view(4096, 4096))
    for h in (0, 13, 31):
        blk = slice(128 * h, 128 * h + 128)
        assert rel(got[blk], ref[blk]) < NS_TOL


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_fused_small_zero_slice(mn, variant):
    U = _seeded(3, 64, 576, 5)
    U[1].zero_()
    _, out, _ = _ns(mn, U, variant=variant)
    assert torch.count_nonzero(out[1]) == 0
    ref = oracle.ns_batched(f64(U), variant)
    for i in (0, 2):
        assert rel(f64(out)[i], ref[i]) < NS_TOL


def test_fused_small_step_captured_in_cuda_graph(mn):
    # Fused launches (cluster attribute), tall transposes and the GEMM path's
    # programmatic dependent launches, captured together and replayed.
    Us = [_seeded(2, 128, 1024, 41), _seeded(2, 700, 96, 42), _seeded(1, 300, 520, 43)]
    outs = []
    bs = []
    for U in Us:
        n, r, c = U.shape
        _, out = _padded(n, r, c, torch.bfloat16, float("nan"))
        outs.append(out)
        bs.append(mn.Batch(n, r, c, ns_in=U, ns_out=out))
    ws = mn.allocate_workspace(bs, -1)
    hp = mn.Hparams()
    mn.muon_ns_batched(bs, hp, ws)          # per-device set-up happens eagerly
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    for o in outs:
        o.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mn.muon_ns_batched(bs, hp, ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for o in outs:
        o.fill_(float("nan"))
    with torch.cuda.graph(g):
        mn.muon_ns_batched(bs, hp, ws, torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    for e, o in zip(eager, outs):
        assert torch.equal(e, o)


def _mixed_batches(mn, seed, with_rows=True):
    # Fused slices (streamed heads, resident conv slices, a tall transposed
    # one) beside GEMM-path slices (short side above 128) in one call.
    shapes = [(8, 128, 4096), (2, 512, 1024), (3, 64, 576), (2, 1024, 512), (2, 700, 96)]
    Us, outs, rss, bs = [], [], [], []
    for k, (n, r, c) in enumerate(shapes):
        U = _seeded(n, r, c, seed + k)
        _, out = _padded(n, r, c, torch.bfloat16, float("nan"))
        rs = torch.full((n, r), float("nan"), dtype=torch.float32, device=DEV) if with_rows else None
        Us.append(U)
        outs.append(out)
        rss.append(rs)
        bs.append(mn.Batch(n, r, c, ns_in=U, ns_out=out, row_sumsq=rs))
    return Us, outs, rss, bs


@pytest.mark.parametrize("variant", ["standard", "gram"])
def test_overlapped_fused_slices_match_single_stream(mn, variant):
    # With both kinds of slices in one call the fused ones run on a second
    # stream beside the GEMM chain; the results (and row sums) are bitwise
    # those of the one-stream schedule, and match the oracle.
    Us, outs, rss, bs = _mixed_batches(mn, 610)
    fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    ws = mn.allocate_workspace(bs, 1 if variant == "standard" else 2)
    results = {}
    for overlap in (1, 0):
        for o, r in zip(outs, rss):
            o.fill_(float("nan"))
            r.fill_(float("nan"))
        with mn.testing_options(overlap=overlap):
            fn(bs, mn.Hparams(), ws)
            torch.cuda.synchronize()
        assert mn.workspace_error(ws) == 0
        results[overlap] = ([o.clone() for o in outs], [r.clone() for r in rss])
    for a, b in zip(results[1][0] + results[1][1], results[0][0] + results[0][1]):
        assert torch.equal(a, b)
    for U, out in zip(Us, outs):
        ref = oracle.ns_batched(f64(U[:1]), variant)
        assert rel(f64(out[:1])[0], ref[0]) < NS_TOL


def test_overlapped_call_is_ordered_before_later_stream_work(mn):
    # Work enqueued on the call's stream right after it (a copy of every
    # output, no host synchronization in between) sees the fused slices'
    # results: the second stream is joined back before the call returns.
    Us, outs, rss, bs = _mixed_batches(mn, 640)
    ws = mn.allocate_workspace(bs, 1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            for o in outs:
                o.fill_(float("nan"))
            mn.muon_ns_batched(bs, mn.Hparams(), ws, s)
            copies = [o.clone() for o in outs] + [r.clone() for r in rss]
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    for c, o in zip(copies, outs + rss):
        assert not torch.isnan(c).any()
        assert torch.equal(c, o)


def test_overlapped_call_first_used_inside_graph_capture(mn):
    # A thread whose first mixed call is inside stream capture makes its
    # second stream and events there; the captured graph replays to the
    # eager result.
    import threading
    Us, outs, rss, bs = _mixed_batches(mn, 670)
    ws = mn.allocate_workspace(bs, 2)
    hp = mn.Hparams()
    with mn.testing_options(overlap=0):
        mn.muon_gram_ns_batched(bs, hp, ws)
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs] + [r.clone() for r in rss]
    box = {}

    def worker():
        try:
            torch.cuda.set_device(0)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                mn.muon_gram_ns_batched(bs, hp, ws, torch.cuda.current_stream())
            for o in outs + rss:
                o.fill_(float("nan"))
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            box["ok"] = True
        except Exception as e:   # reported in the main thread
            box["err"] = e

    t = threading.Thread(target=worker)
    t.start()
    t.join(120)
    assert not t.is_alive()
    assert "err" not in box, box.get("err")
    assert mn.workspace_error(ws) == 0
    for e, o in zip(eager, outs + rss):
        assert torch.equal(e, o)
