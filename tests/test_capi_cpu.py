"""Host-side checks of the C ABI that need no GPU.

The library must load, export every function the public headers declare,
size workspaces, and reject bad arguments before it touches a device.
The calls below pass fake device addresses; every one is built to fail
host-side validation, except one that checks an accepted layout, which runs
only where there is no CUDA device.  The tests that call the device entry
points at all are skipped on a machine with a GPU (the GPU tests cover those
calls with real buffers), so a validation bug can never send a kernel to a
fake address.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_device_present() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # noqa: BLE001
        return False


# Fake device addresses must never reach a device.
no_device = pytest.mark.skipif(_cuda_device_present(), reason="passes fake device addresses: host-only check")


@pytest.fixture(scope="module")
def mn():
    import __graft_entry__
    __graft_entry__._builder().build()
    import newton_schulz_ns_b200 as m
    return m


def _declared():
    names = []
    for h in ("muon_ns.h", "muon_ns_testing.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"MUON_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol(mn):
    from newton_schulz_ns_b200 import _capi
    names = _declared()
    assert set(names) >= {"muon_momentum_norm", "muon_ns_batched", "muon_gram_ns_batched", "normuon_update",
                          "muon_workspace_size"}
    lib = ctypes.CDLL(_capi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert mn.version().count(".") == 2


def test_status_strings(mn):
    from newton_schulz_ns_b200 import _capi
    for s in range(8):
        assert _capi.status_string(s) and _capi.status_string(s) != "unknown status"


def _fake_batch(mn, n, r, c, **kw):
    from newton_schulz_ns_b200 import _capi
    b = _capi.MuonBatch()
    b.n, b.rows, b.cols = n, r, c
    ld = kw.get("ld", c)
    for i, f in enumerate(("grad", "momentum", "ns_in", "ns_out", "weight")):
        v = getattr(b, f)
        base = kw.get("ptr", 0x7F0000000000)
        v.ptr = base + i * 0x10000000 if base else 0
        v.ld = ld
        v.batch_stride = kw.get("bs", r * ld)
        v.dtype = kw.get(f + "_dt", _capi.MUON_BF16)
    b.sumsq = 0x7F0000100000
    b.variance = 0x7F0000200000
    b.fan_out, b.fan_in = r, c
    return b


def _call(mn, fn, batches, ws=None, nbytes=0, hp=None, **kw):
    from newton_schulz_ns_b200 import _capi
    arr = (_capi.MuonBatch * max(1, len(batches)))(*batches)
    h, keep = (hp or mn.Hparams(**kw)).to_c()
    lib = _capi.lib
    if fn == "normuon_update":
        return lib.normuon_update(arr, len(batches), ctypes.byref(h), 1, ws, nbytes, None)
    return getattr(lib, fn)(arr, len(batches), ctypes.byref(h), ws, nbytes, None)


def test_workspace_size_grows_with_batches(mn):
    from newton_schulz_ns_b200 import _capi
    b1 = _fake_batch(mn, 2, 64, 576)
    b2 = _fake_batch(mn, 4, 1024, 512)
    arr1 = (_capi.MuonBatch * 1)(b1)
    arr2 = (_capi.MuonBatch * 2)(b1, b2)
    for which in (0, 1, 2, 3):
        s1 = _capi.lib.muon_workspace_size(arr1, 1, which)
        s2 = _capi.lib.muon_workspace_size(arr2, 2, which)
        assert s1 >= 256 and s2 > s1 and s1 % 256 == 0
    # standard: two m x m bf16 buffers + one X-sized buffer per slice
    ns = _capi.lib.muon_workspace_size(arr2, 2, 1)
    assert ns >= 2 * (2 * 2 * 64 * 64 + 2 * 64 * 576) + 4 * (2 * 2 * 512 * 512 + 2 * 1024 * 512)
    allmax = _capi.lib.muon_workspace_size(arr2, 2, -1)
    assert allmax == max(_capi.lib.muon_workspace_size(arr2, 2, w) for w in range(4))
    assert _capi.lib.muon_workspace_size(arr2, 2, 7) == 0


@no_device
@pytest.mark.parametrize("fn", ["muon_momentum_norm", "muon_ns_batched", "muon_gram_ns_batched", "normuon_update"])
def test_rejects_bad_arguments_before_any_device_work(mn, fn):
    good = _fake_batch(mn, 2, 64, 576)
    # ld smaller than cols
    assert _call(mn, fn, [_fake_batch(mn, 2, 64, 576, ld=500)], 0x7F0000300000, 1 << 30) == 2
    # negative sizes
    assert _call(mn, fn, [_fake_batch(mn, -1, 64, 576)], 0x7F0000300000, 1 << 30) == 2
    # null data pointer
    assert _call(mn, fn, [_fake_batch(mn, 2, 64, 576, ptr=0)], 0x7F0000300000, 1 << 30) == 1
    # workspace: missing, misaligned, too small
    assert _call(mn, fn, [good], None, 0) == 1
    assert _call(mn, fn, [good], 0x7F0000300010, 1 << 30) == 4
    assert _call(mn, fn, [good], 0x7F0000300000, 256) == 5
    # ns_steps out of range and non-finite hyperparameters
    assert _call(mn, fn, [good], 0x7F0000300000, 1 << 30, ns_steps=0) == 1
    assert _call(mn, fn, [good], 0x7F0000300000, 1 << 30, lr=float("nan")) == 1


@no_device
def test_dtype_and_alignment_rules(mn):
    from newton_schulz_ns_b200 import _capi
    # Newton-Schulz operands must be bf16 and meet the 16-byte TMA rule.
    assert _call(mn, "muon_ns_batched", [_fake_batch(mn, 2, 64, 576, ns_in_dt=_capi.MUON_F32)],
                 0x7F0000300000, 1 << 30) == 3
    assert _call(mn, "muon_ns_batched", [_fake_batch(mn, 2, 64, 570, ld=570)], 0x7F0000300000, 1 << 30) == 4
    assert _call(mn, "muon_ns_batched", [_fake_batch(mn, 2, 64, 576, ptr=0x7F0000000008)],
                 0x7F0000300000, 1 << 30) == 4
    # the elementwise calls take f32 or bf16 and any 2-byte-aligned layout
    b = _fake_batch(mn, 2, 64, 570, ld=570, grad_dt=_capi.MUON_F32, momentum_dt=_capi.MUON_F32)
    st = _call(mn, "muon_momentum_norm", [b], 0x7F0000300000, 1 << 30)
    assert st in (6, 7)      # passed validation; no device here (CUDA error) or not a B200


@no_device
@pytest.mark.parametrize("fn", ["muon_ns_batched", "muon_gram_ns_batched"])
def test_newton_schulz_outputs_may_not_overlap_inputs_or_each_other(mn, fn):
    good = _fake_batch(mn, 2, 64, 576)
    # ns_out starting one row into ns_in, or on it
    part = _fake_batch(mn, 2, 64, 576)
    part.ns_out.ptr = part.ns_in.ptr + 2 * 576
    same = _fake_batch(mn, 2, 64, 576)
    same.ns_out.ptr = same.ns_in.ptr
    # another batch's output on this batch's input, and two outputs on one buffer
    other = _fake_batch(mn, 1, 64, 576, ptr=0x7F4000000000)
    other.ns_out.ptr = good.ns_in.ptr + 2 * 576 * 64
    twin = _fake_batch(mn, 1, 64, 576, ptr=0x7F5000000000)
    twin.ns_out.ptr = good.ns_out.ptr
    for bad in ([part], [same], [good, other], [good, twin]):
        assert _call(mn, fn, bad, 0x7F0000300000, 1 << 30) == 1
    # adjacent, not overlapping: passes validation (then no device: CUDA error, or not a B200)
    near = _fake_batch(mn, 2, 64, 576)
    near.ns_out.ptr = near.ns_in.ptr + 2 * (2 * 64 * 576)
    assert _call(mn, fn, [near], 0x7F0000300000, 1 << 30) in (6, 7)


@no_device
def test_empty_batches_enqueue_nothing(mn):
    for fn in ("muon_momentum_norm", "muon_ns_batched", "muon_gram_ns_batched", "normuon_update"):
        assert _call(mn, fn, [_fake_batch(mn, 0, 64, 576)], None, 0) == 0
        assert _call(mn, fn, [_fake_batch(mn, 3, 0, 576)], None, 0) == 0
        assert _call(mn, fn, [], None, 0) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    import subprocess
    import sys
    code = ("import sys, importlib; sys.path.insert(0, %r); import newton_schulz_ns_b200._capi as c; "
            "print('loaded')") % ROOT
    env = dict(os.environ)
    # Point the loader at a copy of the package without the shared object.
    pkg = tmp_path / "newton_schulz_ns_b200"
    pkg.mkdir()
    src = os.path.join(ROOT, "newton_schulz_ns_b200")
    for f in ("__init__.py", "_capi.py"):
        (pkg / f).write_text(open(os.path.join(src, f)).read())
    code = "import sys; sys.path.insert(0, %r); import newton_schulz_ns_b200" % str(tmp_path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env)
    assert r.returncode != 0 and "libmuon_ns.so is missing" in r.stderr


# ----------------------------------------------------------------- Polar Express schedule (host code)

@pytest.mark.parametrize("lower", [1e-4, 1e-3, 1e-2, 0.1, 0.5])
def test_polar_express_schedule_matches_lp_oracle(mn, lower):
    import numpy as np
    import oracle
    got, gerr = mn.polar_express_schedule(lower, 8, safety=1.0)
    # Step by step on the library's own intervals: with safety 1 the image of
    # [lo_t, hi_t] under the minimax quintic is [1 - E_t, 1 + E_t].  (The
    # recursion itself is ill-conditioned for small `lower`: lo_{t+1} = 1 - E_t
    # with E_t close to 1, so two solvers 1e-7 apart in E drift apart later.)
    lo, hi = lower, 1.0
    for t in range(8):
        g = np.array(got[t])
        if hi - lo < 1e-3:
            w = np.array(oracle.FIXED_POINT_QUINTIC)
        else:
            w = np.array(oracle.minimax_quintic_lp(lo, hi)[0])
        # library: Remez exchange in fp64, stored as float32; oracle: LP on a
        # 4001-point grid, whose solver tolerance (~1e-9 on E) moves the
        # coefficients by about that over the interval width cubed (the
        # conditioning of fitting x, x^3, x^5 on a short interval)
        tol = 2e-5 + (2e-9 / (hi - lo) ** 3 if hi - lo >= 1e-3 else 0.0)
        assert np.all(np.abs(g - w) <= tol * np.maximum(1.0, np.abs(w))), (t, g, w)
        mn_, mx_ = oracle.quintic_image(got[t], lo, hi)
        assert abs(max(1 - mn_, mx_ - 1) - gerr[t]) <= 1e-5, (t, mn_, mx_, gerr[t])
        lo, hi = 1.0 - gerr[t], 1.0 + gerr[t]
    if lower >= 1e-3:
        # well-conditioned here: the whole recursion agrees too
        want, werr = oracle.polar_express_lp(lower, 8)
        assert np.allclose(np.array(got), np.array(want), rtol=1e-4, atol=1e-4)
        assert np.allclose(gerr, werr, atol=1e-4)


def test_polar_express_schedule_safety_and_arguments(mn):
    import numpy as np
    (c1,), _ = mn.polar_express_schedule(1e-2, 1, 1.0)
    (c2,), _ = mn.polar_express_schedule(1e-2, 1, 1.02)
    s = 1.02
    assert np.allclose(c2, (c1[0] / s, c1[1] / s ** 3, c1[2] / s ** 5), rtol=1e-6)
    for bad in [dict(lower=0.0), dict(lower=1.0), dict(steps=0), dict(steps=17), dict(safety=0.99),
                dict(safety=2.5)]:
        kw = dict(lower=1e-3, steps=5, safety=1.0)
        kw.update(bad)
        with pytest.raises(mn.MuonError) as e:
            mn.polar_express_schedule(**kw)
        assert e.value.status == 1      # MUON_INVALID_ARG


def test_workspace_holds_the_transposed_copy_of_tall_small_slices(mn):
    # A tall slice with a short side <= 128 that a fused kernel takes runs it
    # on a transposed copy [n][cols][rows] (rows rounded to 64) in the
    # workspace of both Newton-Schulz forms; a wide slice, and a tall one
    # outside those limits, needs none.
    from newton_schulz_ns_b200 import _capi

    def size(b, which):
        return _capi.lib.muon_workspace_size((_capi.MuonBatch * 1)(b), 1, which)

    n, r, c = 3, 700, 96                       # tall, fused
    copy = n * c * ((r + 63) // 64 * 64) * 2
    for which in (1, 2):
        tall = size(_fake_batch(mn, n, r, c), which)
        # the same buffers without the copy: m x m ones of the same m, plus
        # the X-sized buffer of a rows x cols slice (standard: the iterate;
        # Gram: the iterate a restart forms)
        m = c
        mm = n * ((m + 63) // 64 * 64) * m * 2
        base = 256 + 2 * 256                   # error word, norm partials and sums (rounded up)
        xbuf = n * r * ((c + 63) // 64 * 64) * 2
        if which == 1:
            base_bufs = 2 * mm + xbuf
        else:
            base_bufs = 5 * mm + xbuf
        assert tall >= base_bufs + copy
        assert tall - copy < base_bufs + base + 5 * 256 + 8 * n * ((r * c + 8191) // 8192) + 64
    # wide twin, and tall slices the fused kernels do not take (long side past
    # 4096 and not a multiple of 8, or past 16384): no copy
    assert size(_fake_batch(mn, n, c, r), 1) < size(_fake_batch(mn, n, r, c), 1)
    for rows in (5001, 16392):
        t_big = size(_fake_batch(mn, 1, rows, 96), 2)
        assert t_big < (5 * ((96 + 63) // 64 * 64) * 96 * 2 + rows * 128 * 2 + 256 * 8
                        + 4 * ((rows * 96 + 8191) // 8192) + 4096)
    # a tall slice the streaming kernel takes (long side a multiple of 8, past 4096) gets the copy
    t_stream = size(_fake_batch(mn, 1, 5000, 96), 2)
    assert t_stream >= 96 * ((5000 + 63) // 64 * 64) * 2


# ----------------------------------------------------------------- update scale (host code)

@pytest.mark.parametrize("shape,mode,extra", [((4096, 4096), "spectral", 1.0), ((1024, 4096), "spectral", 1.0),
                                              ((8192, 4096), "spectral", 1.0), ((14336, 4096), "spectral", 1.0),
                                              ((4096, 14336), "spectral", 2.5), ((4096, 4096), "rms_norm", 1.0),
                                              ((14336, 4096), "rms_norm", 1.0), ((64, 576), "rms_norm", 0.5),
                                              ((1, 1), "rms_norm", 1.0), ((7168, 2048), "spectral", 0.3)])
def test_update_scale_through_the_c_abi_matches_the_oracle(mn, shape, mode, extra):
    import numpy as np
    import oracle
    got = mn.update_scale(*shape, mode=mode, extra=extra)
    # the ABI takes extra as a float32; the scale is computed in double and rounded once to float32
    want = oracle.update_scale(*shape, mode=mode, extra=float(np.float32(extra)))
    assert got == float(np.float32(want))


def test_update_scale_closed_values(mn):
    import math
    assert mn.update_scale(4096, 4096) == 1.0
    assert mn.update_scale(1024, 4096) == 1.0
    assert abs(mn.update_scale(8192, 4096) - math.sqrt(2)) < 1e-7
    assert abs(mn.update_scale(14336, 4096) - math.sqrt(3.5)) < 1e-7
    assert abs(mn.update_scale(4096, 4096, "rms_norm") - 12.8) < 1e-5
    assert abs(mn.update_scale(1024, 4096, "rms_norm", 0.5) - 6.4) < 1e-5


def test_update_scale_rejects_bad_arguments(mn):
    from newton_schulz_ns_b200 import _capi
    out = ctypes.c_float(0.0)
    for args in [(0, 4, 0, 1.0), (4, 0, 0, 1.0), (-3, 4, 0, 1.0), (4, 4, 2, 1.0), (4, 4, -1, 1.0),
                 (4, 4, 0, float("nan")), (4, 4, 1, float("inf"))]:
        assert _capi.lib.muon_update_scale(*args, ctypes.byref(out)) == 1, args
    assert _capi.lib.muon_update_scale(4, 4, 0, 1.0, None) == 1


@no_device
def test_update_rejects_missing_fans_and_unknown_modes(mn):
    good = _fake_batch(mn, 2, 64, 576)
    nofan = _fake_batch(mn, 2, 64, 576)
    nofan.fan_out = 0
    assert _call(mn, "normuon_update", [nofan], 0x7F0000300000, 1 << 30) == 1
    neg = _fake_batch(mn, 2, 64, 576)
    neg.fan_in = -5
    assert _call(mn, "normuon_update", [neg], 0x7F0000300000, 1 << 30) == 1
    hp = mn.Hparams()
    h, keep = hp.to_c()
    from newton_schulz_ns_b200 import _capi
    arr = (_capi.MuonBatch * 1)(good)
    h.scale_mode = 5
    assert _capi.lib.normuon_update(arr, 1, ctypes.byref(h), 1, 0x7F0000300000, 1 << 30, None) == 1
    h.scale_mode = 0
    h.extra_scale_factor = float("nan")
    assert _capi.lib.normuon_update(arr, 1, ctypes.byref(h), 1, 0x7F0000300000, 1 << 30, None) == 1
    # every call validates the hyperparameters, the restart period included
    for fn in ("muon_momentum_norm", "muon_ns_batched", "muon_gram_ns_batched"):
        assert _call(mn, fn, [good], 0x7F0000300000, 1 << 30, gram_restart=-1) == 1
        assert _call(mn, fn, [good], 0x7F0000300000, 1 << 30, gram_restart=17) == 1
        assert _call(mn, fn, [good], 0x7F0000300000, 1 << 30, scale_mode="spectral", extra_scale_factor=float("inf")) == 1


def test_testing_options_round_trip_and_range_checks(mn):
    from newton_schulz_ns_b200 import _capi

    def now():
        cur = _capi.MuonTestingOptions()
        assert _capi.lib.muon_testing_set_options(None, ctypes.byref(cur)) == 0
        return (cur.fused_small, cur.max_waves, cur.max_problems, cur.pdl, cur.overlap)

    assert now() == (1, 32, 1, 1, 1)
    with mn.testing_options(fused_small=0, max_waves=4, pdl=0, overlap=0):
        assert now() == (0, 4, 1, 0, 0)
    assert now() == (1, 32, 1, 1, 1)
    for bad in [(2, 32, 1, 1, 1), (1, -1, 1, 1, 1), (1, 32, 0, 1, 1), (1, 32, 9, 1, 1), (1, 32, 1, 3, 1),
                (1, 32, 1, 1, 2), (1, 32, 1, 1, -1)]:
        o = _capi.MuonTestingOptions(*bad)
        assert _capi.lib.muon_testing_set_options(ctypes.byref(o), None) == 1
    assert now() == (1, 32, 1, 1, 1)


def test_row_sum_partials_take_workspace_only_when_requested(mn):
    from newton_schulz_ns_b200 import _capi
    n, r, c = 3, 300, 2100
    plain = _fake_batch(mn, n, r, c)
    asked = _fake_batch(mn, n, r, c)
    asked.row_sumsq = 0x7F0000400000
    for which in (1, 2):
        a = _capi.lib.muon_workspace_size((_capi.MuonBatch * 1)(plain), 1, which)
        b = _capi.lib.muon_workspace_size((_capi.MuonBatch * 1)(asked), 1, which)
        # one float per output row and per 128-column half of a 256-column tile (at least 16 per
        # row: the fused path's CTA halves), rounded up to the 256-byte alignment
        per_row = max(2 * ((c + 255) // 256), 16)
        assert b - a == (4 * n * per_row * r + 255) // 256 * 256
