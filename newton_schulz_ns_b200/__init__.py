"""B200-native Muon / NorMuon optimizer step: Python binding of libmuon_ns.

The four calls of the C ABI (include/muon_ns.h) under the same names:
``muon_momentum_norm``, ``muon_ns_batched``, ``muon_gram_ns_batched`` and
``normuon_update``; plus ``muon_workspace_size``.  They take lists of
``Batch`` objects built from torch tensors; torch provides device memory and
streams only.  Every arithmetic step runs in the library's sm_100a kernels.
"""
from __future__ import annotations

import contextlib
import ctypes
import dataclasses
from typing import List, Optional, Sequence

import torch

from . import _capi
from ._capi import MUON_BF16, MUON_F16, MUON_F32, MuonError  # noqa: F401

__all__ = ["Batch", "Hparams", "muon_workspace_size", "muon_momentum_norm", "muon_ns_batched",
           "muon_gram_ns_batched", "normuon_update", "workspace_error", "testing_gemm", "update_scale",
           "ns_flops", "version", "kernel_launches", "muon_momentum_norm_noalloc", "muon_ns_auto_batched",
           "polar_express_schedule", "allocate_workspace", "testing_options", "TwoStreamStep", "MuonError",
           "LIB_PATH"]

LIB_PATH = _capi.LIB_PATH

_DT = {torch.float32: MUON_F32, torch.bfloat16: MUON_BF16, torch.float16: MUON_F16}

QUINTIC = (3.4445, -4.7750, 2.0315)


def version() -> str:
    return _capi.lib.muon_version().decode()


def kernel_launches() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(_capi.lib.muon_kernel_launches())


def polar_express_schedule(lower: float = 1e-3, steps: int = 5, safety: float = 1.01):
    """Per-step (a, b, c) of the Polar Express schedule and each step's max |1 - p| (include/muon_ns.h).

    Host computation in the library; pass the coefficients as
    ``Hparams(ns_steps=steps, abc_schedule=coeffs)``.  The default safety
    factor 1.01 is what bf16 arithmetic needs: with 1.0 a value rounded just
    past the top of the tracked interval meets the steep side of the
    polynomial (a 128 x 1024 Gaussian slice ends 0.13 away from the fp64
    result; with 1.01, 0.02).
    """
    abc = (ctypes.c_float * (3 * steps))()
    err = (ctypes.c_double * steps)()
    st = _capi.lib.muon_polar_express_schedule(float(lower), int(steps), float(safety), abc, err)
    if st != 0:
        raise MuonError(st, "muon_polar_express_schedule")
    coeffs = [(abc[3 * t], abc[3 * t + 1], abc[3 * t + 2]) for t in range(steps)]
    return coeffs, [err[t] for t in range(steps)]


def update_scale(fan_out: int, fan_in: int, mode: str = "spectral", extra: float = 1.0) -> float:
    """The update's shape factor of ONE parameter [fan_out, fan_in], as the library computes it.

    ``mode``: "spectral" or "rms_norm" (include/muon_ns.h, muon_update_scale).
    """
    out = ctypes.c_float(0.0)
    _capi.check(_capi.lib.muon_update_scale(int(fan_out), int(fan_in), _capi.SCALE_MODES[mode], float(extra),
                                            ctypes.byref(out)), "muon_update_scale")
    return float(out.value)


def ns_flops(rows: int, cols: int, variant: str = "standard", steps: int = 5,
             gram_restart: int = _capi.MUON_GRAM_RESTART_DEFAULT) -> float:
    """Floating-point operations the library's kernels perform for one slice.

    Standard: per step X X^T (one triangle, m^2 n), b*A + c*A^2 (one
    triangle, m^3) and B X (2 m^2 n).  Gram: X X^T (m^2 n); per step A^2,
    P Q (except at a segment's first step, where Q = P) and the two factors
    of P A P (except at a segment's last step), each a one-triangle m^3; at
    each restart Q X (2 m^2 n) and X X^T (m^2 n); finally Q X (2 m^2 n).
    """
    m, n = min(rows, cols), max(rows, cols)
    if variant == "standard":
        return float(steps * (3 * m * m * n + m ** 3))
    R = gram_restart

    def restart_at(k):
        return R > 0 and 0 < k < steps and k % R == 0

    prods, restarts, seg = 0, 0, 0
    for k in range(steps):
        if restart_at(k):
            restarts += 1
            seg = k
        prods += 1 + (k != seg) + 2 * (not (k == steps - 1 or restart_at(k + 1)))
    return float(3 * m * m * n + restarts * 3 * m * m * n + prods * m ** 3)


def _view(t: Optional[torch.Tensor], n: int, rows: int, cols: int, name: str) -> _capi.MuonView:
    v = _capi.MuonView()
    if t is None:
        return v
    if t.dim() == 2:
        t = t.unsqueeze(0)
    if t.dim() != 3 or tuple(t.shape) != (n, rows, cols):
        raise ValueError(f"{name}: expected shape {(n, rows, cols)}, got {tuple(t.shape)}")
    if t.stride(2) != 1:
        raise ValueError(f"{name}: rows must be contiguous")
    if t.dtype not in _DT:
        raise ValueError(f"{name}: unsupported dtype {t.dtype}")
    v.ptr = t.data_ptr()
    v.ld = t.stride(1)
    v.batch_stride = t.stride(0) if n > 1 else rows * t.stride(1)
    v.dtype = _DT[t.dtype]
    return v


@dataclasses.dataclass
class Batch:
    """Same-shape slices [n, rows, cols] and the buffers one step touches.

    Tensors are 3-D [n, rows, cols] views (2-D is taken as n = 1) whose rows
    are contiguous; ``sumsq`` is [n], ``variance`` and ``row_sumsq`` [n, rows],
    all fp32.  ``fan_out`` / ``fan_in`` are the shape of the PARAMETER the
    slices come from (shape[0], prod(shape[1:])), which sets the update's
    scale; ``normuon_update`` needs them.
    """
    n: int
    rows: int
    cols: int
    grad: Optional[torch.Tensor] = None
    momentum: Optional[torch.Tensor] = None
    ns_in: Optional[torch.Tensor] = None
    ns_out: Optional[torch.Tensor] = None
    weight: Optional[torch.Tensor] = None
    weight_copy: Optional[torch.Tensor] = None
    sumsq: Optional[torch.Tensor] = None
    variance: Optional[torch.Tensor] = None
    row_sumsq: Optional[torch.Tensor] = None
    fan_out: int = 0
    fan_in: int = 0

    def to_c(self) -> _capi.MuonBatch:
        b = _capi.MuonBatch()
        b.n, b.rows, b.cols = self.n, self.rows, self.cols
        args = (self.n, self.rows, self.cols)
        b.grad = _view(self.grad, *args, "grad")
        b.momentum = _view(self.momentum, *args, "momentum")
        b.ns_in = _view(self.ns_in, *args, "ns_in")
        b.ns_out = _view(self.ns_out, *args, "ns_out")
        b.weight = _view(self.weight, *args, "weight")
        b.weight_copy = _view(self.weight_copy, *args, "weight_copy")
        for name in ("sumsq", "variance", "row_sumsq"):
            t = getattr(self, name)
            if t is not None:
                if t.dtype != torch.float32 or not t.is_contiguous():
                    raise ValueError(f"{name}: contiguous float32 expected")
                want = self.n if name == "sumsq" else self.n * self.rows
                if t.numel() != want:
                    raise ValueError(f"{name}: {want} elements expected, got {t.numel()}")
                setattr(b, name, t.data_ptr())
        b.fan_out, b.fan_in = int(self.fan_out), int(self.fan_in)
        return b


@dataclasses.dataclass
class Hparams:
    mu: float = 0.95
    nesterov: bool = True
    ns_eps: float = 1e-7
    abc: Sequence[float] = QUINTIC
    ns_steps: int = 5
    beta2: float = 0.95
    nor_eps: float = 1e-8
    lr: float = 0.02
    weight_decay: float = 0.0
    abc_schedule: Optional[Sequence[Sequence[float]]] = None
    scale_mode: str = "spectral"
    extra_scale_factor: float = 1.0
    gram_restart: int = _capi.MUON_GRAM_RESTART_DEFAULT

    def to_c(self):
        h = _capi.MuonHparams()
        h.mu, h.nesterov, h.ns_eps = self.mu, int(bool(self.nesterov)), self.ns_eps
        h.a, h.b, h.c = (float(x) for x in self.abc)
        h.ns_steps = int(self.ns_steps)
        h.beta2, h.nor_eps, h.lr, h.weight_decay = self.beta2, self.nor_eps, self.lr, self.weight_decay
        h.scale_mode = _capi.SCALE_MODES[self.scale_mode]
        h.extra_scale_factor = float(self.extra_scale_factor)
        h.gram_restart = int(self.gram_restart)
        keep = None
        if self.abc_schedule is not None:
            flat = [float(v) for row in self.abc_schedule for v in row]
            keep = (ctypes.c_float * len(flat))(*flat)
            h.abc_schedule = ctypes.cast(keep, ctypes.POINTER(ctypes.c_float))
        return h, keep


def _batches(batches: Sequence[Batch]):
    arr = (_capi.MuonBatch * max(1, len(batches)))()
    for i, b in enumerate(batches):
        arr[i] = b.to_c()
    return arr, len(batches)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _ws(workspace: Optional[torch.Tensor]):
    if workspace is None:
        return None, 0
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def muon_workspace_size(batches: Sequence[Batch], which: int = -1) -> int:
    arr, nb = _batches(batches)
    return int(_capi.lib.muon_workspace_size(arr, nb, which))


def allocate_workspace(batches: Sequence[Batch], which: int = -1, device=None) -> torch.Tensor:
    """A uint8 CUDA tensor of muon_workspace_size bytes (torch's allocator aligns it to 512 B).

    Its error word (the first 256 bytes) starts cleared, so workspace_error
    reads 0 for a workspace that no Newton-Schulz call has used yet.
    """
    ws = torch.empty(max(256, muon_workspace_size(batches, which)), dtype=torch.uint8, device=device or "cuda")
    ws[:256].zero_()
    return ws


def muon_momentum_norm(batches: Sequence[Batch], hp: Hparams, workspace: torch.Tensor, stream=None) -> None:
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    p, nbytes = _ws(workspace)
    _capi.check(_capi.lib.muon_momentum_norm(arr, nb, ctypes.byref(h), p, nbytes, _stream_ptr(stream)),
                "muon_momentum_norm")


def muon_momentum_norm_noalloc(batches: Sequence[Batch], hp: Hparams, stream=None) -> None:
    """muon_momentum_norm with the library's static device scratch instead of a workspace.

    For callers that cannot allocate device memory where they run the step.
    Calls that may overlap on the GPU share the scratch and race; the first
    call on a device should come before any stream capture on it.
    """
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    _capi.check(_capi.lib.muon_momentum_norm_noalloc(arr, nb, ctypes.byref(h), _stream_ptr(stream)),
                "muon_momentum_norm_noalloc")


def muon_ns_batched(batches: Sequence[Batch], hp: Hparams, workspace: torch.Tensor, stream=None) -> None:
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    p, nbytes = _ws(workspace)
    _capi.check(_capi.lib.muon_ns_batched(arr, nb, ctypes.byref(h), p, nbytes, _stream_ptr(stream)),
                "muon_ns_batched")


def muon_gram_ns_batched(batches: Sequence[Batch], hp: Hparams, workspace: torch.Tensor, stream=None) -> None:
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    p, nbytes = _ws(workspace)
    _capi.check(_capi.lib.muon_gram_ns_batched(arr, nb, ctypes.byref(h), p, nbytes, _stream_ptr(stream)),
                "muon_gram_ns_batched")


def muon_ns_auto_batched(batches: Sequence[Batch], hp: Hparams, workspace: torch.Tensor, gram_min_ratio: float = 1.25,
                         stream=None) -> None:
    """Newton-Schulz with the Gram form for slices with n >= gram_min_ratio * m, standard otherwise."""
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    p, nbytes = _ws(workspace)
    _capi.check(_capi.lib.muon_ns_auto_batched(arr, nb, ctypes.byref(h), float(gram_min_ratio), p, nbytes,
                                               _stream_ptr(stream)), "muon_ns_auto_batched")


def normuon_update(batches: Sequence[Batch], hp: Hparams, use_normuon: bool, workspace: torch.Tensor,
                   stream=None) -> None:
    arr, nb = _batches(batches)
    h, _keep = hp.to_c()
    p, nbytes = _ws(workspace)
    _capi.check(_capi.lib.normuon_update(arr, nb, ctypes.byref(h), int(bool(use_normuon)), p, nbytes,
                                         _stream_ptr(stream)), "normuon_update")


class TwoStreamStep:
    """One optimizer step over several batches, scheduled on two streams.

    Scheduling only (every operation is one of the C-ABI calls above): the
    Newton-Schulz call of batch i runs on the caller's stream while the
    momentum of batch i + 1 and the NorMuon + update of batch i - 1 run on a
    second stream, so the tensor-core-bound and the HBM-bound kernels of the
    step overlap.  Calls on different streams must not share a workspace:
    each stream gets its own, sized for the largest batch.  Batch i's
    Newton-Schulz call waits for its momentum and its update waits for its
    Newton-Schulz call (events).  The two smallest batches go first and
    last, where their kernels cannot overlap anything.  Results are those of
    the serial calls: every slice's result is independent of the batch it
    is in.

    ``variant``: "standard", "gram" or "auto" (``gram_min_ratio`` as in
    ``muon_ns_auto_batched``).  Call it with the stream to enqueue on (the
    current stream by default); it can be captured in a CUDA graph after one
    eager call.
    """

    def __init__(self, batches: Sequence[Batch], hp: Hparams, variant: str = "standard", use_normuon: bool = True,
                 gram_min_ratio: float = 1.25, device=None):
        if not batches:
            raise ValueError("no batches")
        sizes = [b.n * b.rows * b.cols for b in batches]
        by_size = sorted(range(len(batches)), key=lambda i: (sizes[i], i))
        if len(batches) > 2:
            middle = sorted(by_size[2:], key=lambda i: (-sizes[i], i))
            self.order = [by_size[0]] + middle + [by_size[1]]
        else:
            self.order = by_size
        self.batches = [batches[i] for i in self.order]
        self.hp = hp
        self.variant = variant
        self.use_normuon = bool(use_normuon)
        self.gram_min_ratio = float(gram_min_ratio)
        which_ns = {"standard": 1, "gram": 2, "auto": -1}[variant]
        dev = device or "cuda"
        ns_bytes = max(muon_workspace_size([b], which_ns) for b in self.batches)
        ew_bytes = max(max(muon_workspace_size([b], 0), muon_workspace_size([b], 3)) for b in self.batches)
        self.ws_ns = torch.zeros(max(256, ns_bytes), dtype=torch.uint8, device=dev)
        self.ws_ew = torch.zeros(max(256, ew_bytes), dtype=torch.uint8, device=dev)
        self.ew_stream = torch.cuda.Stream(device=dev)
        self.ev_mom = [torch.cuda.Event() for _ in self.batches]
        self.ev_ns = [torch.cuda.Event() for _ in self.batches]

    def _ns(self, b, stream):
        if self.variant == "standard":
            muon_ns_batched([b], self.hp, self.ws_ns, stream)
        elif self.variant == "gram":
            muon_gram_ns_batched([b], self.hp, self.ws_ns, stream)
        else:
            muon_ns_auto_batched([b], self.hp, self.ws_ns, self.gram_min_ratio, stream)

    def __call__(self, stream=None) -> None:
        main = stream if stream is not None else torch.cuda.current_stream()
        side = self.ew_stream
        side.wait_stream(main)
        bs = self.batches
        for i, b in enumerate(bs):
            muon_momentum_norm([b], self.hp, self.ws_ew, side)
            self.ev_mom[i].record(side)
            main.wait_event(self.ev_mom[i])
            self._ns(b, main)
            self.ev_ns[i].record(main)
            if i > 0:
                side.wait_event(self.ev_ns[i - 1])
                normuon_update([bs[i - 1]], self.hp, self.use_normuon, self.ws_ew, side)
        side.wait_event(self.ev_ns[-1])
        normuon_update([bs[-1]], self.hp, self.use_normuon, self.ws_ew, side)
        main.wait_stream(side)

    def workspace_errors(self) -> int:
        """The Newton-Schulz workspace's error word (0: no device-side wait ran out).

        Each Newton-Schulz call clears the word when it starts, so this is the
        last call's status; the momentum and update kernels have no waits.
        """
        return workspace_error(self.ws_ns)


def workspace_error(workspace: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _capi.check(_capi.lib.muon_workspace_error(workspace.data_ptr(), _stream_ptr(stream), ctypes.byref(out)),
                "muon_workspace_error")
    return int(out.value)


@contextlib.contextmanager
def testing_options(**switches):
    """Temporarily sets the library's kernel-selection switches (include/muon_ns_testing.h).

    Keys: fused_small, max_waves, max_problems, pdl, overlap.  For tests and
    experiments; production calls use the defaults.
    """
    prev = _capi.MuonTestingOptions()
    _capi.check(_capi.lib.muon_testing_set_options(None, ctypes.byref(prev)), "muon_testing_set_options")
    new = _capi.MuonTestingOptions(prev.fused_small, prev.max_waves, prev.max_problems, prev.pdl, prev.overlap)
    for k, v in switches.items():
        if not hasattr(new, k):
            raise KeyError(k)
        setattr(new, k, int(v))
    _capi.check(_capi.lib.muon_testing_set_options(ctypes.byref(new), None), "muon_testing_set_options")
    try:
        yield
    finally:
        _capi.lib.muon_testing_set_options(ctypes.byref(prev), None)


def testing_gemm(A: torch.Tensor, a_mn: bool, B: torch.Tensor, b_mn: bool, C: torch.Tensor, *, K: int,
                 tri: bool = False, D: Optional[torch.Tensor] = None, alpha: float = 1.0, beta: float = 0.0,
                 gamma: float = 0.0, f0: float = 1.0, s_pow: int = 0, sumsq: Optional[torch.Tensor] = None,
                 eps: float = 0.0, row_ss: Optional[torch.Tensor] = None, cta_pair: int = 0,
                 raster_group: int = 0, workspace: torch.Tensor = None, stream=None) -> None:
    """Runs one tensor-core GEMM problem of the library (include/muon_ns_testing.h).

    A, B, C, D are 3-D [slices, rows, cols] with contiguous rows.  C is
    [slices, M, N]; A is [slices, M, K] (a_mn False) or [slices, K, M];
    B is [slices, N, K] (b_mn False) or [slices, K, N].  cta_pair: 0 the
    library's choice, 1 single-CTA tiles, 2 CTA-pair tiles.
    """
    S, M, N = C.shape
    if A.dtype != B.dtype:
        raise ValueError("A and B must share a dtype")

    def ld_bs(t):
        return (t.stride(1), t.stride(0)) if t is not None else (0, 0)

    lda, bsa = ld_bs(A)
    ldb, bsb = ld_bs(B)
    ldc, bsc = ld_bs(C)
    ldd, bsd = ld_bs(D)
    p, nbytes = _ws(workspace)
    st = _capi.lib.muon_testing_gemm(
        M, N, K, S, int(tri), _DT[A.dtype],
        A.data_ptr(), lda, bsa, int(a_mn), B.data_ptr(), ldb, bsb, int(b_mn),
        D.data_ptr() if D is not None else None, ldd, bsd, _DT[D.dtype] if D is not None else MUON_BF16,
        C.data_ptr(), ldc, bsc, _DT[C.dtype], alpha, beta, gamma, f0, s_pow,
        sumsq.data_ptr() if sumsq is not None else None, eps,
        row_ss.data_ptr() if row_ss is not None else None, int(cta_pair), int(raster_group), p, nbytes,
        _stream_ptr(stream))
    _capi.check(st, "muon_testing_gemm")
