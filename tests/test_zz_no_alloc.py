"""muon_momentum_norm_noalloc: the momentum call for callers that cannot allocate.

Some callers run the optimizer step where they may not allocate device
memory (a runtime that owns all of it, a replay or real-time loop) and have
nowhere to keep a workspace.  This entry point keeps its scratch in a static
device array inside the library instead.  It must produce what
muon_momentum_norm produces from the same inputs, call after call.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

DEV = "cuda"


def _cuda_device_present() -> bool:
    try:
        return torch.cuda.is_available()
    except Exception:  # noqa: BLE001
        return False


@pytest.fixture(scope="module")
def mn():
    import newton_schulz_ns_b200 as m
    return m


def _state(shapes, seed):
    g = torch.Generator().manual_seed(seed)
    out = []
    for (n, r, c, gdt, mdt) in shapes:
        G = (torch.randn((n, r, c), generator=g)).to(gdt).to(DEV)
        M = (torch.randn((n, r, c), generator=g) * 0.5).to(mdt).to(DEV)
        out.append((G, M))
    return out


def _batches(mn, state):
    bs = []
    for G, M in state:
        n, r, c = G.shape
        bs.append(mn.Batch(n, r, c, grad=G, momentum=M,
                           ns_in=torch.full((n, r, c), float("nan"), dtype=torch.bfloat16, device=DEV),
                           sumsq=torch.full((n,), float("nan"), device=DEV)))
    return bs


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_twice_in_a_row(mn):
    shapes = [(3, 64, 576, torch.bfloat16, torch.bfloat16), (2, 300, 200, torch.float32, torch.float32),
              (1, 37, 51, torch.bfloat16, torch.float32)]
    base = _state(shapes, 1)
    ref = _batches(mn, [(G.clone(), M.clone()) for G, M in base])
    new = _batches(mn, [(G.clone(), M.clone()) for G, M in base])
    hp = mn.Hparams(mu=0.95, nesterov=True)
    ws = mn.allocate_workspace(ref, 0)
    for call in range(2):
        mn.muon_momentum_norm(ref, hp, ws)
        mn.muon_momentum_norm_noalloc(new, hp)
        torch.cuda.synchronize()
        for a, b in zip(ref, new):
            # Same kernels and reduction order: the results agree exactly, which
            # is inside every tolerance the parity tests use.
            assert torch.equal(a.momentum, b.momentum), call
            assert torch.equal(a.ns_in, b.ns_in), call
            assert torch.equal(a.sumsq, b.sumsq), call
            assert bool(torch.all(torch.isfinite(b.sumsq)))


@pytest.mark.gpu
def test_noalloc_many_batches_match_workspace_call(mn):
    # More batches than one elementwise launch takes (16): the call is split
    # into several launches, each with its own stretch of the shared scratch.
    shapes = [(1 + k % 3, 16 + 8 * k, 40 + 24 * (k % 5), torch.bfloat16, torch.bfloat16 if k % 2 else torch.float32)
              for k in range(37)]
    base = _state(shapes, 2)
    ref = _batches(mn, [(G.clone(), M.clone()) for G, M in base])
    new = _batches(mn, [(G.clone(), M.clone()) for G, M in base])
    hp = mn.Hparams(mu=0.9, nesterov=True)
    ws = mn.allocate_workspace(ref, 0)
    for call in range(2):
        mn.muon_momentum_norm(ref, hp, ws)
        mn.muon_momentum_norm_noalloc(new, hp)
        torch.cuda.synchronize()
        for a, b in zip(ref, new):
            assert torch.equal(a.momentum, b.momentum), call
            assert torch.equal(a.ns_in, b.ns_in), call
            assert torch.equal(a.sumsq, b.sumsq), call


# The call below passes fake device addresses that host-side validation must
# reject; like the other fake-address checks it never runs where a GPU is.
@pytest.mark.skipif(_cuda_device_present(), reason="passes fake device addresses: host-only check")
def test_noalloc_rejects_calls_beyond_its_scratch(mn):
    from newton_schulz_ns_b200 import _capi
    b = _capi.MuonBatch()
    b.n, b.rows, b.cols = 9, 32768, 32768              # 9 * 131072 chunks of 8192 elements > 2**20
    for i, f in enumerate(("grad", "momentum", "ns_in")):
        v = getattr(b, f)
        v.ptr = 0x7F0000000000 + i * 0x100000000
        v.ld = 32768
        v.batch_stride = 32768 * 32768
        v.dtype = _capi.MUON_BF16
    b.sumsq = 0x7F0100000000
    arr = (_capi.MuonBatch * 1)(b)
    h, _keep = mn.Hparams().to_c()
    st = _capi.lib.muon_momentum_norm_noalloc(arr, 1, ctypes.byref(h), None)
    assert st == 5, _capi.status_string(st)               # MUON_WORKSPACE_TOO_SMALL, nothing enqueued
