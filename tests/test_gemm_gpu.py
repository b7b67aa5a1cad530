"""The tcgen05 GEMM of the library against a float64 matrix product.

Each case runs one GEMM problem through the C ABI's test hook on slices that
span several 128x256 tiles with ragged tails, in every operand-major
combination the Newton-Schulz calls use, and checks the epilogue terms
(alpha, addend, identity, per-slice norm factor, row sums of squares).
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def mn():
    import newton_schulz_ns_b200 as m
    return m


def _ws():
    return torch.zeros(256, dtype=torch.uint8, device=DEV)


def _rnd(shape, dtype, seed, scale=1.0):
    """Seeded N(0, scale^2) [S, R, C] on the device, rows padded to a multiple of 8 elements (TMA rule)."""
    g = torch.Generator().manual_seed(seed)
    S, R, C = shape
    ld = (C + 7) // 8 * 8
    x = torch.zeros((S, R, ld), dtype=dtype, device=DEV)
    x[:, :, :C] = (torch.randn(shape, generator=g) * scale).to(dtype).to(DEV)
    return x[:, :, :C]


def _empty(shape, dtype, fill=float("nan")):
    S, R, C = shape
    ld = (C + 7) // 8 * 8
    return torch.full((S, R, ld), fill, dtype=dtype, device=DEV)[:, :, :C]


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _check(C, ref, rel_tol=4e-3):
    C = _f64(C)
    err = np.linalg.norm(C - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err < rel_tol, f"relative error {err:.3e}"
    assert np.max(np.abs(C - ref)) <= 2e-2 * np.max(np.abs(ref)) + 1e-6


PAIRS = [1, 2]      # single-CTA 128x256 tiles, 2-CTA (cta_group::2) 256x256 tiles


@pytest.mark.parametrize("cta_pair", PAIRS)
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K,S", [(300, 520, 200, 2), (128, 256, 64, 1), (77, 40, 33, 3), (513, 300, 520, 1)])
def test_gemm_majors(mn, a_mn, b_mn, dtype, M, N, K, S, cta_pair):
    A = _rnd((S, K, M) if a_mn else (S, M, K), dtype, 1)
    B = _rnd((S, K, N) if b_mn else (S, N, K), dtype, 2)
    C = _empty((S, M, N), torch.bfloat16)
    ws = _ws()
    mn.testing_gemm(A, bool(a_mn), B, bool(b_mn), C, K=K, alpha=0.5, cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    a = _f64(A)
    b = _f64(B)
    a = np.swapaxes(a, 1, 2) if a_mn else a                 # [S, M, K]
    b = b if b_mn else np.swapaxes(b, 1, 2)                 # [S, K, N]
    _check(C, 0.5 * a @ b)


@pytest.mark.parametrize("cta_pair", PAIRS)
def test_gemm_strided_slices_and_padding(mn, cta_pair):
    # Slices with ld > cols and batch stride > rows*ld; padding must stay untouched.
    S, M, N, K = 3, 200, 260, 136
    Abig = _rnd((S, M + 8, K + 24), torch.bfloat16, 3)
    A = Abig[:, :M, :K]
    Bbig = _rnd((S, K, N + 44), torch.bfloat16, 4)
    B = Bbig[:, :, :N]
    Cbig = torch.full((S, M + 5, N + 60), 7.0, dtype=torch.bfloat16, device=DEV)
    C = Cbig[:, :M, :N]
    ws = _ws()
    mn.testing_gemm(A, False, B, True, C, K=K, cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    _check(C, _f64(A) @ _f64(B))
    rest = _f64(Cbig)
    rest[:, :M, :N] = 7.0
    assert np.all(rest == 7.0)


@pytest.mark.parametrize("cta_pair", PAIRS)
@pytest.mark.parametrize("mnmaj", [0, 1])
@pytest.mark.parametrize("m,n", [(384, 500), (200, 1000), (64, 576), (513, 130), (1024, 600)])
def test_syrk_triangle_mirror(mn, mnmaj, m, n, cta_pair):
    S = 2
    X = _rnd((S, n, m) if mnmaj else (S, m, n), torch.bfloat16, 5)
    C = _empty((S, m, m), torch.bfloat16)
    ss = torch.tensor([4.0, 9.0], device=DEV)
    ws = _ws()
    mn.testing_gemm(X, bool(mnmaj), X, bool(mnmaj), C, K=n, tri=True, s_pow=2, sumsq=ss, eps=0.0, f0=3.0,
                    cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    x = _f64(X)
    x = np.swapaxes(x, 1, 2) if mnmaj else x
    ref = x @ np.swapaxes(x, 1, 2) * 3.0 / np.array([4.0, 9.0])[:, None, None]
    Cn = _f64(C)
    assert np.array_equal(Cn, np.swapaxes(Cn, 1, 2))        # mirror is exact
    _check(C, ref)


@pytest.mark.parametrize("cta_pair", PAIRS)
def test_symmetric_epilogue_addend_identity_fp16(mn, cta_pair):
    # P = a I + (b/k) A + (c/k^2) A A with fp16 A, as the Gram iteration forms it.
    S, m = 2, 300
    X = _rnd((S, m, 2 * m), torch.float32, 6)
    A32 = X @ X.transpose(1, 2) / (2 * m)
    A = _empty((S, m, m), torch.float16, 0.0)
    A.copy_(A32.to(torch.float16))
    P = _empty((S, m, m), torch.float16)
    a, b, c, k = 3.4445, -4.7750, 2.0315, 4.0
    ws = _ws()
    mn.testing_gemm(A, False, A, False, P, K=m, tri=True, D=A, alpha=c / k ** 2, beta=b / k, gamma=a,
                    cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    an = _f64(A)
    ref = a * np.eye(m)[None] + (b / k) * an + (c / k ** 2) * an @ an
    _check(P, ref, rel_tol=2e-3)


@pytest.mark.parametrize("cta_pair", PAIRS)
def test_row_sums_of_squares(mn, cta_pair):
    S, M, N, K = 2, 260, 600, 100
    A = _rnd((S, M, K), torch.bfloat16, 7)
    B = _rnd((S, K, N), torch.bfloat16, 8)
    C = _empty((S, M, N), torch.bfloat16)
    nh = 2 * ((N + 255) // 256)                 # one partial per 128-column half of a 256-column tile
    rss = torch.full((S, nh, M), float("nan"), device=DEV)
    ws = _ws()
    mn.testing_gemm(A, False, B, True, C, K=K, row_ss=rss, cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    c = _f64(C)
    for t in range(nh):
        ref = np.sum(c[:, :, 128 * t:128 * (t + 1)] ** 2, axis=2)
        assert np.allclose(_f64(rss)[:, t], ref, rtol=1e-5)


@pytest.mark.parametrize("cta_pair", PAIRS)
def test_gemm_deterministic_and_batch_invariant(mn, cta_pair):
    M, N, K = 384, 512, 640
    A = _rnd((4, M, K), torch.bfloat16, 9)
    B = _rnd((4, K, N), torch.bfloat16, 10)
    ws = _ws()
    C1 = torch.empty((4, M, N), dtype=torch.bfloat16, device=DEV)
    C2 = torch.empty_like(C1)
    mn.testing_gemm(A, False, B, True, C1, K=K, cta_pair=cta_pair, workspace=ws)
    mn.testing_gemm(A, False, B, True, C2, K=K, cta_pair=cta_pair, workspace=ws)
    C3 = torch.empty((1, M, N), dtype=torch.bfloat16, device=DEV)
    mn.testing_gemm(A[2:3], False, B[2:3], True, C3, K=K, cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)
    assert torch.equal(C1[2:3], C3)


def test_pair_and_single_cta_agree(mn):
    # Same products, different tile shapes: the accumulation order over K is
    # the same, so the two kernels produce the same bits.
    M, N, K = 640, 768, 512
    A = _rnd((2, M, K), torch.bfloat16, 11)
    B = _rnd((2, K, N), torch.bfloat16, 12)
    ws = _ws()
    C1 = _empty((2, M, N), torch.bfloat16)
    C2 = _empty((2, M, N), torch.bfloat16)
    mn.testing_gemm(A, False, B, True, C1, K=K, cta_pair=1, workspace=ws)
    mn.testing_gemm(A, False, B, True, C2, K=K, cta_pair=2, workspace=ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    _check(C2, _f64(A) @ _f64(B))
    assert float((C1.float() - C2.float()).abs().max()) <= 2e-2 * float(C1.float().abs().max())


def test_bounded_wait_times_out_and_context_survives(mn):
    # A device wait that nothing satisfies gives up after its limit, reports
    # through the workspace word, and leaves the context usable.
    from newton_schulz_ns_b200 import _capi
    ws = _ws()
    st = _capi.lib.muon_testing_bounded_wait(2_000_000, ws.data_ptr(), 256, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert mn.workspace_error(ws) == 4                      # MUON_TESTING_WAIT_TIMEOUT
    A = _rnd((1, 128, 64), torch.bfloat16, 13)
    B = _rnd((1, 256, 64), torch.bfloat16, 14)
    C = _empty((1, 128, 256), torch.bfloat16)
    mn.testing_gemm(A, False, B, False, C, K=64, workspace=ws)
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0
    _check(C, _f64(A) @ np.swapaxes(_f64(B), 1, 2))


@pytest.mark.parametrize("cta_pair", PAIRS)
def test_long_k_launch_with_several_waves(mn, cta_pair):
    # K > 2048 and more tiles than one wave: the launch keeps one epilogue
    # warp per TMEM lane quadrant (short-K or single-wave launches split each
    # tile's columns over two).  Addend, per-slice factor and row sums, as
    # the Newton-Schulz apply phase uses them.
    S, M, N, K = 2, 2048, 2600, 2304
    A = _rnd((S, M, K), torch.bfloat16, 21, 0.05)
    B = _rnd((S, K, N), torch.bfloat16, 22, 0.05)
    D = _rnd((S, M, N), torch.bfloat16, 23)
    C = _empty((S, M, N), torch.bfloat16)
    ss = torch.tensor([4.0, 9.0], device=DEV)
    nh = 2 * ((N + 255) // 256)
    rss = torch.full((S, nh, M), float("nan"), device=DEV)
    ws = _ws()
    mn.testing_gemm(A, False, B, True, C, K=K, D=D, alpha=1.0, beta=0.75, f0=1.0, s_pow=1, sumsq=ss, eps=0.0,
                    row_ss=rss, cta_pair=cta_pair, workspace=ws)
    torch.cuda.synchronize()
    f = np.array([1 / 2.0, 1 / 3.0])[:, None, None]
    ref = f * (_f64(A) @ _f64(B) + 0.75 * _f64(D))
    _check(C, ref)
    c = _f64(C)
    for t in range(nh):
        want = np.sum(c[:, :, 128 * t:128 * (t + 1)] ** 2, axis=2)
        assert np.allclose(_f64(rss)[:, t], want, rtol=1e-5)


@pytest.mark.parametrize("tri", [False, True])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0)])
def test_single_and_pair_tiles_are_bitwise_equal(mn, tri, a_mn, b_mn):
    # Both tile kernels issue the same K-ordered sequence of K = 16 tensor-core
    # steps into fp32 accumulators and share the epilogue, so the choice of
    # kernel (single-CTA 128 x 256 or 2-CTA 256 x 256 tiles) never changes a
    # stored bit; the library may pick either for a slice.
    S, M, K = 2, 520, 700
    N = M if tri else 1000
    A = _rnd((S, K, M) if a_mn else (S, M, K), torch.bfloat16, 21)
    B = A if tri else _rnd((S, K, N) if b_mn else (S, N, K), torch.bfloat16, 22)
    bmn = a_mn if tri else b_mn
    D = _rnd((S, M, N), torch.bfloat16, 23)
    ss = torch.tensor([2.0, 5.0], device=DEV)
    rows = {}
    outs = {}
    for pair in PAIRS:
        C = _empty((S, M, N), torch.bfloat16)
        rss = None if tri else torch.full((S, 2 * ((N + 255) // 256), M), float("nan"), device=DEV)
        mn.testing_gemm(A, bool(a_mn), B, bool(bmn), C, K=K, tri=tri, D=D, alpha=0.7, beta=1.3, gamma=0.25,
                        s_pow=1, sumsq=ss, eps=1e-7, row_ss=rss, cta_pair=pair, workspace=_ws())
        torch.cuda.synchronize()
        outs[pair] = C.clone()
        rows[pair] = rss
    assert torch.equal(outs[1], outs[2])
    if not tri:
        assert torch.equal(rows[1], rows[2])
