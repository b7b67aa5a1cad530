"""Newton-Schulz on seeded random shapes, all in one call, against the fp64 oracle.

Sixteen shapes drawn once from a fixed seed (log-uniform sides from 1 to
1536, wide and tall, 1 to 3 slices, row strides padded past the columns)
and seven chosen ones (the fused kernels' limits, streamed slices, GEMM-path
shapes over one and several 256-blocks)
go through one `muon_ns_batched` / `muon_gram_ns_batched` call, so the
fused small-side kernels (resident and streamed, with and without the
transposed copy) run on the second stream beside the tensor-core GEMM
path.  Bars: 3e-2 relative Frobenius error per slice against the oracle;
nothing written outside a slice; every batch bit for bit equal to the same
batch called alone; the row sums of squares equal to those of the stored
output (1e-5 relative).
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
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _shapes(count=16, seed=2026):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        r, c = (int(np.exp(rng.uniform(0.0, np.log(1536.0)))) for _ in range(2))
        if min(r, c) > 640:             # keeps the fp64 oracle at seconds per slice
            continue
        out.append((int(rng.integers(1, 4)), max(r, 1), max(c, 1)))
    # The fused kernels' limits, streamed slices, and GEMM-path shapes of one
    # and several 256-blocks (compact symmetric storage, ragged tiles).
    out += [(2, 128, 2600), (1, 3000, 96), (1, 129, 700), (2, 256, 1000), (1, 600, 600), (1, 1400, 300),
            (1, 513, 770)]
    return out


SHAPES = _shapes()


def _batch(mn, n, r, c, seed, pad):
    g = torch.Generator().manual_seed(seed)
    ld = (c + 7) // 8 * 8 + pad
    U = torch.zeros((n, r, ld), dtype=torch.bfloat16, device=DEV)[:, :, :c]
    U.copy_(torch.randn((n, r, c), generator=g).to(torch.bfloat16).to(DEV))
    base = torch.full((n, r, ld), float("nan"), dtype=torch.bfloat16, device=DEV)
    rs = torch.full((n, r), float("nan"), dtype=torch.float32, device=DEV)
    return U, base, base[:, :, :c], rs


def _caller(mn, variant):
    if variant == "auto":   # Gram for slices with n >= 1.25 m, standard otherwise
        return lambda bs, hp, ws: mn.muon_ns_auto_batched(bs, hp, ws, 1.25)
    return mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched


def _oracle_variant(variant, r, c):
    if variant != "auto":
        return variant
    m, n = min(r, c), max(r, c)
    return "gram" if n > m and n >= 1.25 * m else "standard"


@pytest.mark.parametrize("variant", ["standard", "gram", "auto"])
def test_random_shapes_one_call(mn, variant):
    fn = _caller(mn, variant)
    parts = [_batch(mn, n, r, c, 900 + k, 8 * (k % 3)) for k, (n, r, c) in enumerate(SHAPES)]
    bs = [mn.Batch(U.shape[0], U.shape[1], U.shape[2], ns_in=U, ns_out=o, row_sumsq=rs)
          for U, _, o, rs in parts]
    ws = mn.allocate_workspace(bs, -1)
    fn(bs, mn.Hparams(), ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    together = [(o.clone(), rs.clone()) for _, _, o, rs in parts]
    for (U, base, o, rs), (n, r, c) in zip(parts, SHAPES):
        assert torch.isnan(base[:, :, c:].float()).all(), (n, r, c)      # nothing past the slice
        got = f64(o)
        ref = oracle.ns_batched(f64(U), _oracle_variant(variant, r, c))
        for i in range(n):
            assert rel(got[i], ref[i]) < NS_TOL, ((n, r, c), i, rel(got[i], ref[i]))
        ss = (got.astype(np.float64) ** 2).sum(axis=2)
        np.testing.assert_allclose(f64(rs), ss, rtol=1e-5, atol=1e-30)
    # Each batch alone: the same bits (no result depends on the rest of the call).
    for k in (0, 5, len(SHAPES) - 3, len(SHAPES) - 1):
        U, _, o, rs = parts[k]
        o.fill_(float("nan"))
        rs.fill_(float("nan"))
        w1 = mn.allocate_workspace([bs[k]], -1)
        fn([bs[k]], mn.Hparams(), w1)
        torch.cuda.synchronize()
        assert mn.workspace_error(w1) == 0
        assert torch.equal(o, together[k][0]) and torch.equal(rs, together[k][1]), SHAPES[k]
