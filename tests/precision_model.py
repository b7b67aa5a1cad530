"""A numpy model of the storage precision of the CUDA Newton-Schulz path.

Test helper, not an oracle of the method: the fp64 oracle under oracle/ is
the method.  This model runs the same iteration with every stored matrix
rounded to bf16 (round-to-nearest-even) and every product accumulated in
float64 before rounding to float32, which is what bf16 tensor-core operands
with fp32 accumulation compute up to summation order.  It is used only where
the storage precision and the exact method legitimately part ways (rank-
deficient inputs, whose null space collects rounding noise that the
iteration amplifies; slices with a very short side, whose few singular
values sit where the composed quintic is steep), to check that the device
does no worse than that arithmetic.  The fused small-side kernels store
their standard-form iterates in fp16 (`ns_standard_f16`), the GEMM path in
bf16 (`ns_standard_bf16`).
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


def _f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float16).astype(np.float64)


def ns_standard_f16(U, steps=5, eps=1e-7, abc=(3.4445, -4.7750, 2.0315)):
    """Standard iteration of the fused small-side kernels (short side <= 128).

    X0 = fp16(s * bf16(U)) with s = 1 / (||U||_F + eps) in float32; then X, A
    and B = b A + c A^2 stored in fp16 between products (fp32 accumulation),
    the last X in bf16.
    """
    a, b, c = abc
    X = np.asarray(U, dtype=np.float64)
    tr = X.shape[0] > X.shape[1]
    if tr:
        X = X.T
    Xb = _bf16(X)
    s = float(np.float32(1.0) / (np.sqrt(np.float32(np.sum(Xb * Xb))) + np.float32(eps)))
    Xh = _f16(_f32(s * Xb))
    for k in range(steps):
        A = _f16(_f32(Xh @ Xh.T))
        B = _f16(_f32(c * _f32(A @ A) + b * A))
        Y = _f32(_f32(B @ Xh) + a * Xh)
        Xh = _bf16(Y) if k == steps - 1 else _f16(Y)
    return Xh.T if tr else Xh


def ns_gram_f16(U, steps=5, eps=1e-7, abc=(3.4445, -4.7750, 2.0315), restart=3, kappa=16384.0):
    """Gram iteration with the library's storage precisions.

    The m x m iterates are stored in fp16 with A kept as kappa*A (kappa = 2^14
    keeps A's O(1/m) entries out of fp16's subnormal range); a Q that goes
    into a product with the m x n side is stored in bf16, as are X and O.
    Restarts (every `restart` steps) form X = f Q X in bf16 and start again
    from A = kappa X X^T, Q = I.
    """
    a, b, c = abc
    X = np.asarray(U, dtype=np.float64)
    tr = X.shape[0] > X.shape[1]
    if tr:
        X = X.T
    X = _bf16(X)
    m = X.shape[0]
    s = 1.0 / (np.sqrt(np.sum(X * X)) + eps)
    I = np.eye(m)
    Ah = _f16(_f32(X @ X.T) * (kappa * s * s))
    f = s                                  # X's factor: s while X is the unnormalized input
    Q = None

    def restart_at(k):
        return restart > 0 and 0 < k < steps and k % restart == 0

    for k in range(steps):
        if restart_at(k):
            X = _bf16(f * _f32(Q @ X))
            f = 1.0
            Ah = _f16(_f32(X @ X.T) * kappa)
            Q = None
        end = k == steps - 1 or restart_at(k + 1)
        Pm = _f32(c / (kappa * kappa) * _f32(Ah @ Ah) + b / kappa * Ah) + a * I
        if Q is None:
            Q = _bf16(Pm) if end else _f16(Pm)
            P = Q
        else:
            P = _f16(Pm)
            Q = (_bf16 if end else _f16)(P @ Q)
        if not end:
            R = _f16(P @ Ah)
            Ah = _f16(P @ R)
    O = _bf16(f * _f32(Q @ X))
    return O.T if tr else O
