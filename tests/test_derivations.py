"""Numerical checks, in numpy fp64 on random data, of the two identities the
CUDA backward relies on (CPU only; no oracle or CUDA code involved).

For strictly-lower A, T = (I + A)^-1, and Delta defined by
(I + A) Delta = U - Kc S (the chunk equation of "Gated DeltaNet-2", LIT-802
review, Key takeaways 2), the chain rule through W = T Kc, U' = T U and
Delta = U' - W S gives dT = dW Kc^T + dDelta U^T with dW = -dDelta S^T, and:
  (1) -T^T dT T^T = -(T^T dDelta) Delta^T   (so dA needs no C x C x C product)
  (2) T^T dW = -(T^T dDelta) S^T
"""

import numpy as np


def test_gradient_of_the_inverse_collapses():
    rng = np.random.default_rng(7)
    C, dk, dv = 24, 10, 7
    A = np.tril(rng.normal(size=(C, C)), -1) * 0.2
    T = np.linalg.inv(np.eye(C) + A)
    Kc = rng.normal(size=(C, dk))
    U = rng.normal(size=(C, dv))
    S = rng.normal(size=(dk, dv))
    Delta = T @ U - T @ Kc @ S
    np.testing.assert_allclose((np.eye(C) + A) @ Delta, U - Kc @ S, atol=1e-12)
    dDelta = rng.normal(size=(C, dv))
    dW = -dDelta @ S.T
    dT = dW @ Kc.T + dDelta @ U.T
    lhs = -T.T @ dT @ T.T
    dU = T.T @ dDelta
    np.testing.assert_allclose(lhs, -dU @ Delta.T, atol=1e-11)
    np.testing.assert_allclose(T.T @ dW, -dU @ S.T, atol=1e-11)
