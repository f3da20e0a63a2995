"""The chunk-local algebra of the tensor-core prefill, written out in numpy fp64
in the kernel's own form and checked against the oracle's chunk form (O2) on the
CPU.

The kernel forms the key and query scores of a 64-token chunk per 16-row block.
Off-diagonal blocks (rows in block R, keys in block J < R) are products of two
factors that are each at most 1: the row factor exp(g_r - gb_R) and the key
version exp(gb_R - g_i), gb_R being the cumulative log decay through the row
before block R.  A diagonal block uses its own reference gb_R, so its key factor
can exceed 1; when the block's decay range exceeds 80 nats it is formed pairwise
instead, walking i down from r with the decay prod_{i < j <= r} alpha_j carried
as a running product already multiplied into k_r and q_r.  This test writes
both forms out, requires them to equal the plain definition
sum_c k_rc k_ic exp(g_rc - g_ic), and requires U = T beta V and
Wk = T beta K exp(g) built from them to match the oracle's intermediates: a
wrong reference, a factor on the wrong side or an off-by-one in the running
product fails it without a GPU.
"""
import numpy as np
import pytest

import oracle

RANGE_MAX = 80.0   # nats: a diagonal block beyond it is formed pairwise


def scores_kernel_form(kk, qq, la):
    """A (keys x keys, strictly lower) and P (queries x keys, lower with the
    diagonal) of one chunk, L <= 64 rows, as the kernel forms them."""
    L, d = kk.shape
    g = np.cumsum(la, axis=0)
    nb = (L + 15) // 16
    gb = np.zeros((nb + 1, d))                     # gb[R]: through the row before block R
    for R in range(1, nb + 1):
        gb[R] = g[min(16 * R, L) - 1]
    A = np.zeros((L, L))
    P = np.zeros((L, L))
    for R in range(nb):
        rows = slice(16 * R, min(16 * R + 16, L))
        ke = kk[rows] * np.exp(g[rows] - gb[R])    # row factors, <= 1
        qe = qq[rows] * np.exp(g[rows] - gb[R])
        for J in range(R):                          # off-diagonal: key versions referenced to block R
            cols = slice(16 * J, 16 * J + 16)
            kv = kk[cols] * np.exp(gb[R] - g[cols])     # <= 1
            A[rows, cols] = ke @ kv.T
            P[rows, cols] = qe @ kv.T
        n = rows.stop - rows.start
        if np.max(gb[R] - g[rows.stop - 1]) <= RANGE_MAX:
            kv = kk[rows] * np.exp(gb[R] - g[rows])     # the diagonal block's own version (>= 1)
            A[rows, rows] = np.tril(ke @ kv.T, -1)
            P[rows, rows] = np.tril(qe @ kv.T)
        else:                                           # pairwise, running products
            alpha = np.exp(la[rows])
            for r in range(n):
                fa, fp = kk[rows][r].copy(), qq[rows][r].copy()
                for i in range(r, -1, -1):
                    if i < r:
                        fa = fa * alpha[i + 1]
                        fp = fp * alpha[i + 1]
                        A[rows.start + r, rows.start + i] = fa @ kk[rows][i]
                    P[rows.start + r, rows.start + i] = fp @ kk[rows][i]
    return A, P, g


def scores_definition(kk, qq, la):
    g = np.cumsum(la, axis=0)
    E = np.exp(np.minimum(g[:, None, :] - g[None, :, :], 0.0))
    A = np.tril(np.einsum('rc,ic,ric->ri', kk, kk, E), -1)
    P = np.tril(np.einsum('rc,ic,ric->ri', qq, kk, E))
    return A, P


def _inputs(L, regime, seed):
    rng = np.random.default_rng(seed)
    d, dv = 16, 8
    kk = rng.standard_normal((L, d)) / np.sqrt(d)
    qq = rng.standard_normal((L, d)) / np.sqrt(d)
    vv = rng.standard_normal((L, dv))
    beta = rng.uniform(0.0, 1.0, L)
    if regime == "near1":
        la = -rng.uniform(0.0, 1e-3, (L, d))
    elif regime == "near0":                   # every diagonal block beyond 80 nats
        la = -8.0 - 8.0 * rng.uniform(0.0, 1.0, (L, d))
    else:                                      # channels of both kinds: some blocks flagged
        la = np.where(rng.uniform(size=(L, d)) < 0.5, -rng.uniform(0.0, 0.1, (L, d)),
                      -rng.uniform(3.0, 12.0, (L, d)))
    return kk, qq, vv, beta, la


@pytest.mark.parametrize("regime", ["near1", "near0", "mixed"])
@pytest.mark.parametrize("L", [64, 37, 16, 1])
def test_kernel_scores_equal_the_definition(L, regime):
    kk, qq, _, _, la = _inputs(L, regime, seed=L)
    A, P, _ = scores_kernel_form(kk, qq, la)
    A0, P0 = scores_definition(kk, qq, la)
    scale = max(np.max(np.abs(A0)), np.max(np.abs(P0)))
    np.testing.assert_allclose(A, A0, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(P, P0, rtol=0, atol=1e-12 * scale)


@pytest.mark.parametrize("regime", ["near1", "near0", "mixed"])
def test_kernel_form_gives_the_oracle_u_and_wk(regime):
    """U = (I + beta A)^-1 beta V and Wk = (I + beta A)^-1 beta K exp(g) of every
    chunk of a 150-token sequence (two full chunks and a ragged one), from the
    kernel-form scores, against O2's intermediates."""
    T, C = 150, 64
    kk, qq, vv, beta, la = _inputs(T, regime, seed=7)
    ref = oracle.chunkform(qq[:, None], kk[:, None], vv[:, None], la[:, None], beta[:, None],
                           np.array([0, T]), C, intermediates=True)
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        A, _, g = scores_kernel_form(kk[sl], qq[sl], la[sl])
        b = beta[sl]
        Tm = np.linalg.inv(np.eye(len(b)) + b[:, None] * A)
        U = Tm @ (b[:, None] * vv[sl])
        Wk = Tm @ (b[:, None] * kk[sl] * np.exp(g))
        np.testing.assert_allclose(U, ref["u"][sl, 0], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(Wk, ref["wk"][sl, 0], rtol=1e-9, atol=1e-12)


def test_running_product_in_fp32_stays_within_its_rounding_bound():
    """In fp32 the factor prod_{i < j <= 15} alpha_j built by the walk carries at
    most 14 product roundings (relative error <= 14 * 2^-24 to first order)
    against the same alphas multiplied exactly, whatever the decay range (here
    up to 75 nats, inside fp32's normal range)."""
    rng = np.random.default_rng(3)
    alpha = np.exp(-3.0 - 2.0 * rng.uniform(size=(16, 32))).astype(np.float32)
    f = np.ones(32, np.float32)
    worst = 0.0
    for i in range(14, -1, -1):
        f = (f * alpha[i + 1]).astype(np.float32)
        exact = np.prod(alpha[i + 1:].astype(np.float64), axis=0)
        worst = max(worst, float(np.max(np.abs(f.astype(np.float64) - exact) / exact)))
    assert worst <= 14.5 * 2.0 ** -24
