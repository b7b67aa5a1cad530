"""A numpy model of the float32 arithmetic of the elementwise kernels.

Test helper, not an oracle of the method (the fp64 oracle under oracle/ is
the method).  The momentum kernel evaluates, per element and in float32 with
fused multiply-adds (one rounding each):
    M_new = fl32(mu*M + G),   U = bf16(fl32(mu*M_new + G))   (Nesterov)
and the update kernel
    W_new = fl32(-coef*O + fl32(W*keep)),   keep = fl32(1 - lr*wd)
with coef the float32 per-row coefficient lr*scale*factor*d_row.  The model
repeats those roundings; a float32 fused multiply-add is emulated in float64
(the product of two float32 values is exact there, the sum is rounded once
more before the float32 rounding, which differs from a single rounding only
when the sum lies within 2^-53 of a float32 tie: rare enough to allow a
couple of such elements in a test).  It is used to count how often float32
arithmetic of the stated formulas rounds to a different bf16 value than the
exact (fp64) result does, and to check that the device computes exactly
that arithmetic.  It shares no code with the CUDA library.
"""
import numpy as np


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16(x):
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def fma32(a, b, c):
    """float32 fused multiply-add of float32 inputs (emulated, see the module note)."""
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def momentum_f32(G, M, mu, nesterov=True, mom_store="f32"):
    """(stored M_new, bf16 U) as the momentum kernel computes them from float32/bf16 inputs."""
    mu = float(np.float32(mu))
    mn = fma32(mu, M, G)
    u = fma32(mu, mn, G) if nesterov else mn
    return (bf16(mn) if mom_store == "bf16" else mn), bf16(u)


def update_f32(W, O, coef, lr, wd, w_store="f32"):
    """W_new as the update kernel computes it, given the float32 per-element coefficient."""
    keep = f32(1.0 - f32(float(np.float32(lr)) * float(np.float32(wd))))
    w = fma32(-f32(coef), O, f32(np.asarray(W, np.float64) * keep))
    return bf16(w) if w_store == "bf16" else w


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (the smallest subnormal spacing at 0)."""
    ax = np.abs(np.asarray(x, np.float64))
    ulp = np.abs(bf16(ax * (1 + 2.0 ** -7)) - bf16(ax))
    return np.maximum(ulp, 2.0 ** -133)
