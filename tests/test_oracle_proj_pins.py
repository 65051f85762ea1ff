"""Pins of the oracle's projection (P[m, n] = sum_k W[m, k] X[n, k], laid out channel-major
[B, rows, L] or token-major [Ntok, M]) against a brute-force sum and known weights."""
import numpy as np

import oracle


def test_brute_force_small():
    rng = np.random.default_rng(0)
    M, K, B, L = 5, 7, 3, 4
    W, X = rng.standard_normal((M, K)), rng.standard_normal((B * L, K))
    x0, x1 = oracle.proj(W, X, L, M0=2)
    tm = oracle.proj(W, X, L, token_major=True)
    for m in range(M):
        for b in range(B):
            for t in range(L):
                s = 0.0
                for k in range(K):
                    s += W[m, k] * X[b * L + t, k]
                got = x0[b, m, t] if m < 2 else x1[b, m - 2, t]
                assert abs(got - s) <= 1e-12 * (1 + abs(s))
                assert abs(tm[b * L + t, m] - s) <= 1e-12 * (1 + abs(s))


def test_permutation_weights_move_features():
    """W = a row permutation of the identity: output channel m is input feature perm[m] of
    each token, so the channel-major result is X transposed per sample, rows permuted."""
    rng = np.random.default_rng(1)
    K, B, L = 6, 2, 5
    perm = rng.permutation(K)
    W = np.eye(K)[perm]
    X = rng.standard_normal((B * L, K))
    x0, x1 = oracle.proj(W, X, L)
    assert x1 is None
    want = X.reshape(B, L, K).transpose(0, 2, 1)[:, perm]
    assert np.array_equal(x0, want)
