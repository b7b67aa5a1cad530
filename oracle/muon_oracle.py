"""Plain fp64 CPU oracle of the Muon / NorMuon optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library and imports nothing from it.

Everything is numpy float64, one matrix at a time, with no blocking, fusion
or reordering beyond what the method states.  Storage rounding (bf16 or fp32
buffers that the optimizer writes back) is emulated with this module's own
round-to-nearest-even routines, at the points where the optimizer stores.

Sources (titles of the pages the method is taken from):

* [dion-121] microsoft/dion PR #121, "Fix convolution flattening in megabatches
  and NorMuon normalization".
* [mcore-lsm] Megatron-Core API docs, ``core.optimizer.layer_sharded_muon``.
* [ds-8437] DeepSpeed issue #8437, "Muon under AutoTP orthogonalizes each shard,
  so the update depends on the TP degree".

Readings taken where the pages leave a step open (each is listed in the
design notes, with its reason):

* momentum is ``M <- mu*M + G`` and the Nesterov input is ``U = G + mu*M``;
* Frobenius normalization divides by ``||X||_F + eps``;
* a slice with more rows than columns is iterated transposed (tie: not);
* the quintic coefficients are the same at every iteration;
* the X update of the standard iteration is ``X <- a*X + B@X``;
* the Gram variant iterates the polynomial on ``X0 X0^T`` and applies the
  accumulated factor to ``X0`` once at the end;
* the NorMuon variance is the mean of squares along the row (no centering),
  the normalization divides by ``sqrt(v) + eps``, no bias correction, zero
  initial variance, and the rescale restores the slice's pre-normalization
  Frobenius norm (a zero result stays zero);
* the update scale is ``sqrt(max(1, fan_out/fan_in)) * extra``, from the
  parameter's own (fan_out, fan_in); weight decay is decoupled and applied
  before the update.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

QUINTIC_ABC = (3.4445, -4.7750, 2.0315)

__all__ = [
    "QUINTIC_ABC", "bf16_round", "fp32_round", "momentum_nesterov", "frobenius_normalize",
    "newton_schulz", "gram_newton_schulz", "ns_batched", "per_head_ns", "flatten_megabatch",
    "normuon_normalize", "spectral_scale", "rms_norm_scale", "update_scale", "weight_update", "muon_step_slices",
    "ns_flops",
]


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

def fp32_round(x) -> np.ndarray:
    """Round float64 values to the nearest float32 (IEEE RN-even), back as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_round(x) -> np.ndarray:
    """Round float64 values to bfloat16, round-to-nearest-even, back as float64.

    bfloat16 keeps the top 16 bits of an IEEE float32.  Rounding from float64
    goes through float32 first, which is what a float32 value stored as bf16
    sees; the float32 step is exact for every value the optimizer stores in
    bf16, because those values are computed in float32 on the device.  NaN is
    not produced by the optimizer and is not handled.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return fp32_round(x)
    if dtype == "bf16":
        return bf16_round(x)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# ---------------------------------------------------------------------------
# step 1: momentum with Nesterov look-ahead
# ---------------------------------------------------------------------------

def momentum_nesterov(G: np.ndarray, M: np.ndarray, mu: float, nesterov: bool = True,
                      mom_store: str = "f64") -> Tuple[np.ndarray, np.ndarray]:
    """Momentum buffer update and the Newton-Schulz input.

    [mcore-lsm] ``LayerShardedMuon``: momentum 0.95 and ``nesterov=True`` by
    default; its ``step()`` starts with the elementwise momentum update "as in
    base Muon".  Reading: ``M <- mu*M + G``; with Nesterov the orthogonalized
    input is ``U = G + mu*M_new``, else ``U = M_new``.  ``U`` is formed from the
    unrounded new momentum; ``mom_store`` only rounds the buffer written back.
    """
    G = np.asarray(G, dtype=np.float64)
    M = np.asarray(M, dtype=np.float64)
    m_new = mu * M + G
    u = G + mu * m_new if nesterov else m_new.copy()
    return _store(m_new, mom_store), u


# ---------------------------------------------------------------------------
# step 2-4: Newton-Schulz orthogonalization
# ---------------------------------------------------------------------------

def frobenius_normalize(X: np.ndarray, eps: float) -> np.ndarray:
    """[ds-8437] "Why it happens": both kernels first divide by the matrix norm.

    Reading: ``X / (||X||_F + eps)``.
    """
    X = np.asarray(X, dtype=np.float64)
    return X / (np.sqrt(np.sum(X * X)) + eps)


def _orient(U: np.ndarray) -> Tuple[np.ndarray, bool]:
    """Iterate on the short side: a slice with more rows than columns is transposed."""
    U = np.asarray(U, dtype=np.float64)
    if U.ndim != 2:
        raise ValueError("Newton-Schulz takes one 2-D slice")
    if U.shape[0] > U.shape[1]:
        return U.T, True
    return U, False


def _step_coefs(abc, steps: int):
    """Per-step (a, b, c): one triple for every step, or one triple per step.

    A per-step schedule is what the Polar Express iteration uses (named in
    [dion-121] "Validation"); the quintic of the Megatron-Core docs is the
    same triple at every step.
    """
    abc = list(abc)
    if len(abc) == 3 and not hasattr(abc[0], "__len__"):
        return [tuple(float(v) for v in abc)] * steps
    if len(abc) < steps:
        raise ValueError("schedule shorter than the step count")
    return [tuple(float(v) for v in t) for t in abc[:steps]]


def newton_schulz(U: np.ndarray, steps: int = 5, eps: float = 1e-7,
                  abc: Sequence[float] = QUINTIC_ABC) -> np.ndarray:
    """Standard quintic Newton-Schulz of one slice, result in the slice's orientation.

    [ds-8437] "Why it happens": normalize, then iterate on ``X @ X.mT``.
    [mcore-lsm] ``use_syrk``: the two symmetric products are ``A = X X^T`` and
    ``B = b*A + c*A^2``; ``coefficient_type='quintic'``, ``num_ns_steps=5``.
    Each step then forms ``X <- a*X + B @ X``.  ``abc`` is one (a, b, c) for
    every step or a per-step schedule.
    """
    X, transposed = _orient(U)
    X = frobenius_normalize(X, eps)
    for a, b, c in _step_coefs(abc, steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if transposed else X


def gram_newton_schulz(U: np.ndarray, steps: int = 5, eps: float = 1e-7,
                       abc: Sequence[float] = QUINTIC_ABC, restart: int = 0) -> np.ndarray:
    """Gram Newton-Schulz of one slice: the same map, iterated on the small side.

    [ds-8437] "Why it happens" / "Measurement": the Gram kernel also
    normalizes and works from ``X @ X.mT``, and gives the same shard numbers
    as the standard kernel.  The pages give no algorithm text; reading: with
    ``X0`` normalized and ``G = X0 X0^T`` (m x m), keep ``A = G`` and ``Q = I``
    and repeat ``P = a*I + b*A + c*A^2``, ``Q <- P Q``, ``A <- P A P``; the
    result is ``Q X0``.  Because every matrix here is a polynomial in ``G``
    they commute, ``X_k = Q_k X0`` and ``X_k X_k^T = Q_k G Q_k``, so this equals
    the standard iteration in exact arithmetic (also with a per-step
    schedule of (a, b, c)).

    ``restart = R > 0``: before steps R, 2R, ... the iterate ``X = Q X`` is
    formed and the iteration starts again from it (``A = X X^T``, ``Q = I``).
    By the same identities this changes nothing in exact arithmetic; it is the
    reading the library takes to keep low-precision iterates of ``A`` from
    drifting (rank-deficient slices), and it is kept here so that the oracle
    computes the same sequence of products.
    """
    X, transposed = _orient(U)
    X = frobenius_normalize(X, eps)
    m = X.shape[0]
    I = np.eye(m)
    A = X @ X.T
    Q = I.copy()
    for k, (a, b, c) in enumerate(_step_coefs(abc, steps)):
        if restart and k > 0 and k % restart == 0:
            X = Q @ X
            A = X @ X.T
            Q = I.copy()
        P = a * I + b * A + c * (A @ A)
        Q = P @ Q
        A = P @ A @ P
    O = Q @ X
    return O.T if transposed else O


def ns_batched(U: np.ndarray, variant: str = "standard", steps: int = 5, eps: float = 1e-7,
               abc: Sequence[float] = QUINTIC_ABC, restart: int = 0) -> np.ndarray:
    """Newton-Schulz of every slice of a [N, rows, cols] megabatch, one slice at a time.

    [dion-121] "Problem and fix": a megabatch is orthogonalized per slice
    [N, out, prod(rest)], never across slices.  ``restart`` applies to the
    Gram variant only.
    """
    U = np.asarray(U, dtype=np.float64)
    if U.ndim != 3:
        raise ValueError("megabatch must be [N, rows, cols]")
    if variant not in ("standard", "gram"):
        raise ValueError(f"unknown variant {variant!r}")
    out = np.empty_like(U)
    for i in range(U.shape[0]):
        if variant == "standard":
            out[i] = newton_schulz(U[i], steps=steps, eps=eps, abc=abc)
        else:
            out[i] = gram_newton_schulz(U[i], steps=steps, eps=eps, abc=abc, restart=restart)
    return out


def per_head_ns(W: np.ndarray, heads: int, variant: str = "standard", steps: int = 5,
                eps: float = 1e-7, abc: Sequence[float] = QUINTIC_ABC) -> np.ndarray:
    """Per-head Newton-Schulz of a head-blocked projection [heads*d, cols].

    [ds-8437] "What could be done", option 3: split dim 0 into head blocks and
    orthogonalize each block on its own.
    """
    W = np.asarray(W, dtype=np.float64)
    r, c = W.shape
    if r % heads:
        raise ValueError("rows must divide into heads")
    blocks = W.reshape(heads, r // heads, c)
    return ns_batched(blocks, variant, steps, eps, abc).reshape(r, c)


def flatten_megabatch(X: np.ndarray) -> np.ndarray:
    """[N, out, *rest] -> [N, out, prod(rest)] ([dion-121] "Problem and fix")."""
    X = np.asarray(X)
    if X.ndim < 3:
        raise ValueError("megabatch needs a stack axis and an output axis")
    return X.reshape(X.shape[0], X.shape[1], -1)


# ---------------------------------------------------------------------------
# step 5: NorMuon normalization
# ---------------------------------------------------------------------------

def normuon_normalize(O: np.ndarray, v: np.ndarray, beta2: float, eps: float
                      ) -> Tuple[np.ndarray, np.ndarray]:
    """NorMuon on one [rows, cols] slice in the parameter's orientation.

    [dion-121] follow-on "What it does": one variance per output channel (row
    of the flattened matrix), computed over the last dim; "Compatibility":
    the rescale is norm-preserving and local to the slice.
    Steps: ``v <- beta2*v + (1-beta2)*mean_j O_ij^2``; ``Oh = O / (sqrt(v)+eps)``
    per row; ``Oh *= ||O||_F / ||Oh||_F`` (left at zero when ``Oh`` is zero).
    Returns (Oh, v_new).
    """
    O = np.asarray(O, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64).reshape(-1)
    if O.ndim != 2 or v.shape[0] != O.shape[0]:
        raise ValueError("O must be [rows, cols] and v [rows]")
    if O.shape[1] == 0:
        return O.copy(), v.copy()
    ms = np.mean(O * O, axis=1)
    v_new = beta2 * v + (1.0 - beta2) * ms
    Oh = O / (np.sqrt(v_new) + eps)[:, None]
    n_o = math.sqrt(float(np.sum(O * O)))
    n_oh = math.sqrt(float(np.sum(Oh * Oh)))
    if n_oh > 0.0:
        Oh = Oh * (n_o / n_oh)
    return Oh, v_new


# ---------------------------------------------------------------------------
# step 6: update
# ---------------------------------------------------------------------------

def spectral_scale(fan_out: int, fan_in: int, extra: float = 1.0) -> float:
    """Shape factor of the update, from one PARAMETER's (fan_out, fan_in).

    [dion-121] review "Correctness — confirmed": the LR adjustment uses
    ``fan_out = shape[0]`` and ``fan_in = prod(shape[1:])`` of a single
    parameter; [mcore-lsm] ``scale_mode='spectral'``, ``extra_scale_factor``.
    Reading: ``sqrt(max(1, fan_out/fan_in)) * extra``.
    """
    return math.sqrt(max(1.0, fan_out / fan_in)) * extra


def rms_norm_scale(fan_out: int, fan_in: int, extra: float = 1.0) -> float:
    """Shape factor of the ``rms_norm`` mode: ``0.2 * sqrt(max(fan_out, fan_in)) * extra``.

    The pages name the mode ([dion-121] review: ``adjust_lr_rms_norm``;
    [mcore-lsm] ``scale_mode``) but print no formula.  Reading: the RMS
    matching of Liu et al., "Muon is Scalable for LLM Training" (2025): an
    orthogonalized m x n update (m <= n, unit singular values) has element
    RMS ``1/sqrt(n)``, so this factor gives it RMS 0.2 -- a typical AdamW
    update's -- whatever the shape.
    """
    return 0.2 * math.sqrt(max(fan_out, fan_in)) * extra


def update_scale(fan_out: int, fan_in: int, mode: str = "spectral", extra: float = 1.0) -> float:
    """The update's shape factor of one parameter in the given ``scale_mode``."""
    if fan_out < 1 or fan_in < 1:
        raise ValueError("fan_out and fan_in must be positive")
    if mode == "spectral":
        return spectral_scale(fan_out, fan_in, extra)
    if mode == "rms_norm":
        return rms_norm_scale(fan_out, fan_in, extra)
    raise ValueError(f"unknown scale mode {mode!r}")


def weight_update(W: np.ndarray, Oh: np.ndarray, lr: float, weight_decay: float,
                  scale: float, store: str = "f64") -> np.ndarray:
    """Decoupled weight decay then ``W -= lr * scale * Oh``, rounded once on store.

    [mcore-lsm] ``use_decoupled_weight_decay=True``; ``_apply_update``: one
    multiply-add in the promoted precision and one downcast on store.
    """
    W = np.asarray(W, dtype=np.float64)
    return _store(W * (1.0 - lr * weight_decay) - lr * scale * np.asarray(Oh, np.float64), store)


# ---------------------------------------------------------------------------
# whole step over a list of same-shape slices
# ---------------------------------------------------------------------------

def muon_step_slices(G: np.ndarray, M: np.ndarray, W: np.ndarray, v: Optional[np.ndarray], *,
                     mu: float = 0.95, nesterov: bool = True, ns_eps: float = 1e-7,
                     ns_steps: int = 5, abc: Sequence[float] = QUINTIC_ABC,
                     variant: str = "standard", restart: int = 0, normuon: bool = False, beta2: float = 0.95,
                     nor_eps: float = 1e-8, lr: float = 0.02, weight_decay: float = 0.0,
                     lr_scale: float = 1.0, mom_store: str = "f64", w_store: str = "f64",
                     O_override: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """One Muon / NorMuon step over a [N, rows, cols] group of slices.

    ``lr_scale`` is the update's shape factor of the PARAMETER the slices come
    from (``spectral_scale`` of its own shape).  ``O_override`` replaces the
    Newton-Schulz result, so that the later stages can be checked on exactly
    the orthogonalized matrices another implementation produced.
    Returns M (stored), U, O, Oh, v (or None), W (stored).
    """
    G = np.asarray(G, np.float64)
    M_new, U = momentum_nesterov(G, M, mu, nesterov, mom_store)
    if O_override is None:
        O = ns_batched(U, variant, ns_steps, ns_eps, abc, restart)
    else:
        O = np.asarray(O_override, np.float64)
    Oh = np.empty_like(O)
    v_new = None
    if normuon:
        v_new = np.empty((O.shape[0], O.shape[1]), np.float64)
        for i in range(O.shape[0]):
            Oh[i], v_new[i] = normuon_normalize(O[i], v[i], beta2, nor_eps)
    else:
        Oh[...] = O
    W_new = weight_update(W, Oh, lr, weight_decay, lr_scale, w_store)
    return {"M": M_new, "U": U, "O": O, "Oh": Oh, "v": v_new, "W": W_new}


def ns_flops(m: int, n: int, variant: str = "standard", steps: int = 5,
             triangle: bool = True, restart: int = 0) -> float:
    """Floating-point operations of one slice's orthogonalization (m <= n).

    Standard, full products: per step ``2m^2n`` (X X^T) + ``2m^3`` (A^2) +
    ``2m^2n`` (B X).  With one triangle of the two symmetric products
    ([mcore-lsm] ``use_syrk``): ``m^2n + m^3 + 2m^2n``.  Gram, triangle
    products: ``m^2n`` for ``G`` and ``2m^2n`` for the final ``Q X``, plus per
    step a triangle ``m^3`` for each of ``A^2``, ``P Q`` (none on a segment's
    first step, where Q = P), and the two factors of ``P A P`` (none on a
    segment's last step, whose A is never used); a restart adds ``Q X``
    (``2m^2n``) and ``X X^T`` (``m^2n``, one triangle).
    """
    m, n = min(m, n), max(m, n)
    if variant == "standard":
        per = (m * m * n + m ** 3 + 2 * m * m * n) if triangle else (4 * m * m * n + 2 * m ** 3)
        return float(steps * per)
    if variant == "gram":
        def restart_at(k):
            return bool(restart) and 0 < k < steps and k % restart == 0
        prods, restarts, seg = 0, 0, 0
        for k in range(steps):
            if restart_at(k):
                restarts += 1
                seg = k
            prods += 1                                                     # A^2
            prods += 0 if k == seg else 1                                  # P Q
            prods += 0 if (k == steps - 1 or restart_at(k + 1)) else 2     # P (P A)
        per_prod = m ** 3 if triangle else 2 * m ** 3
        gram = m * m * n * (1 if triangle else 2)
        return float(gram + 2 * m * m * n + restarts * (gram + 2 * m * m * n) + prods * per_prod)
    raise ValueError(variant)
