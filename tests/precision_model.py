"""A numpy model of the storage precision of the CUDA Newton-Schulz path.

Test helper, not an oracle of the method: the fp64 oracle under oracle/ is
the method.  This model runs the same iteration with every stored matrix
rounded to bf16 (round-to-nearest-even) and every product accumulated in
float64 before rounding to float32, which is what bf16 tensor-core operands
with fp32 accumulation compute up to summation order.  It is used only where
bf16 arithmetic and the exact method legitimately part ways (rank-deficient
inputs, whose null space collects rounding noise that the iteration
amplifies), to check that the device does no worse than that arithmetic.
It shares no code with the CUDA library.
"""
import numpy as np


def _bf16(x):
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def ns_standard_bf16(U, steps=5, eps=1e-7, abc=(3.4445, -4.7750, 2.0315)):
    """Standard iteration with bf16 storage of X, A = X X^T and B = b A + c A^2."""
    a, b, c = abc
    X = np.asarray(U, dtype=np.float64)
    tr = X.shape[0] > X.shape[1]
    if tr:
        X = X.T
    Xb = _bf16(X)
    s = 1.0 / (np.sqrt(np.sum(Xb * Xb)) + eps)
    for k in range(steps):
        A = _bf16(_f32((s * s if k == 0 else 1.0) * (Xb @ Xb.T)))
        B = _bf16(_f32(c * _f32(A @ A) + b * A))
        Xb = _bf16(_f32((s if k == 0 else 1.0) * (_f32(B @ Xb) + a * Xb)))
    return Xb.T if tr else Xb
