"""The chunkwise backward algebra the CUDA kernels implement, checked in fp64
against the oracle's token-level reverse mode (O3) on the CPU.

The pages give no backward pass; the kernels use a derivation of their own
(the chunk map is affine in its start state, T = (I + A)^-1 is applied
transposed by back substitution, dA = -(Y U^T + Z Wk^T), and dlog alpha_j sums
exactly the terms whose decay spans token j).  This test writes those
formulas out with numpy on small inputs, chunk by chunk, and requires the
gradients of O3 to 1e-10: a wrong sign, transpose or index in the derivation
fails it without a GPU.
"""
import numpy as np
import pytest

import oracle


def chunk_backward(q, k, v, la, beta, s0, do, dfs, C):
    """One sequence, one head: q, k, la [T, dk], v [T, dv], beta [T], s0, dfs
    [dk, dv], do [T, dv].  Returns dq, dk, dv, dla, dbeta, ds0."""
    T, dk = q.shape
    chunks = [(c0, min(C, T - c0)) for c0 in range(0, T, C)]
    # forward, keeping what the backward reads
    S = s0.copy()
    saved = []
    for c0, L in chunks:
        sl = slice(c0, c0 + L)
        qq, kk, vv, b, g = q[sl], k[sl], v[sl], beta[sl], np.cumsum(la[sl], axis=0)
        E = np.exp(np.minimum(g[:, None, :] - g[None, :, :], 0.0))        # [r, i, c], used for i <= r
        low, inc = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
        At = np.einsum('rc,ic,ric->ri', kk, kk, E) * low
        P = np.einsum('rc,ic,ric->ri', qq, kk, E) * inc
        Tm = np.linalg.inv(np.eye(L) + b[:, None] * At)
        Kg, Qg, Kd = kk * np.exp(g), qq * np.exp(g), kk * np.exp(g[-1] - g)
        U, Wk = Tm @ (b[:, None] * vv), Tm @ (b[:, None] * Kg)
        W = U - Wk @ S
        saved.append(dict(sl=sl, g=g, E=E, At=At, P=P, Tm=Tm, Kg=Kg, Qg=Qg, Kd=Kd, U=U, Wk=Wk, W=W, S=S.copy(),
                          b=b, low=low, inc=inc, kk=kk, qq=qq, vv=vv))
        S = np.exp(g[-1])[:, None] * S + Kd.T @ W
    # reverse chain: dW = P^T dO + Kd dS', dS = Diag(Gam) dS' + Qg^T dO - Wk^T dW
    dS = dfs.copy()
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dla", la), ("dbeta", beta))}
    for s in reversed(saved):
        dOc = do[s["sl"]]
        dSe = dS
        dW = s["P"].T @ dOc + s["Kd"] @ dSe
        dS = np.exp(s["g"][-1])[:, None] * dSe + s["Qg"].T @ dOc - s["Wk"].T @ dW
        # chunk-parallel part
        dQg = dOc @ s["S"].T
        dKd = s["W"] @ dSe.T
        dWk = -dW @ s["S"].T
        dGam = np.sum(dSe * s["S"], axis=1)
        dP = (dOc @ s["W"].T) * s["inc"]
        Y = s["Tm"].T @ dW                       # (I + A)^T Y = dW
        Z = s["Tm"].T @ dWk
        b = s["b"]
        dA = -(Y @ s["U"].T + Z @ s["Wk"].T) * s["low"]
        dAt = b[:, None] * dA
        out["dv"][s["sl"]] = b[:, None] * Y
        dKg = b[:, None] * Z
        out["dbeta"][s["sl"]] = np.sum(s["vv"] * Y, 1) + np.sum(s["Kg"] * Z, 1) + np.sum(dA * s["At"], 1)
        kk, qq, E, g = s["kk"], s["qq"], s["E"], s["g"]
        L = len(b)
        x1 = np.einsum('ri,ic,ric->rc', dAt, kk, E)
        x2 = np.einsum('ri,ic,ric->rc', dP, kk, E)
        y = np.einsum('ri,rc,ric->ic', dAt, kk, E) + np.einsum('ri,rc,ric->ic', dP, qq, E)
        out["dq"][s["sl"]] = x2 + dQg * np.exp(g)
        out["dk"][s["sl"]] = x1 + y + dKg * np.exp(g) + dKd * np.exp(g[-1] - g)
        # dlog alpha_j: pairwise terms with i < j <= r, Qg/Kg terms of rows r >= j,
        # Kd terms of rows r < j, and the Gamma term
        Tp = (dAt[:, :, None] * kk[:, None, :] + dP[:, :, None] * qq[:, None, :]) * kk[None, :, :] * E
        dla = np.zeros((L, dk))
        for j in range(L):
            dla[j] = Tp[j:, :j].sum(axis=(0, 1))
            dla[j] += ((dQg * s["Qg"] + dKg * s["Kg"])[j:]).sum(axis=0)
            dla[j] += ((dKd * s["Kd"])[:j]).sum(axis=0)
            dla[j] += dGam * np.exp(g[-1])
        out["dla"][s["sl"]] = dla
    out["ds0"] = dS
    return out


@pytest.mark.parametrize("T,C", [(23, 8), (40, 16), (7, 64)])
def test_chunk_backward_algebra_matches_token_reverse_mode(T, C):
    rng = np.random.default_rng(T * 100 + C)
    dk, dv = 6, 5
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    la = -np.logaddexp(0.0, rng.standard_normal((T, dk)) + 1.0)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    s0 = rng.standard_normal((dk, dv))
    do = rng.standard_normal((T, dv))
    dfs = rng.standard_normal((dk, dv))
    got = chunk_backward(q, k, v, la, beta, s0, do, dfs, C)
    ref = oracle.backward(q[:, None], k[:, None], v[:, None], la[:, None], beta[:, None], [0, T], do[:, None],
                          d_final_state=dfs[None, None], init_state=s0[None, None])
    pairs = (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dla", "dlog_alpha"), ("dbeta", "dbeta"))
    for mine, theirs in pairs:
        np.testing.assert_allclose(got[mine], ref[theirs][:, 0], rtol=1e-9, atol=1e-10, err_msg=mine)
    np.testing.assert_allclose(got["ds0"], ref["d_init_state"][0, 0], rtol=1e-9, atol=1e-10)


def tile_assembled_F(T):
    """F(j) = sum_{r >= j} sum_{i < j} T[r, i] (T: [64, 64], lower triangle used)
    assembled from 4 x 4 tile sums the way the CUDA backward does it: for
    j = 4m + u, the tiles of row blocks a > m add their sums left of column
    block m plus their first u column sums; row block m adds, over its tiles
    left of the diagonal, the rows u..3, and its diagonal tile the pairs
    y < u <= x."""
    L = T.shape[0]
    nb = L // 4
    F = np.zeros(L)
    for a in range(nb):
        rs = np.zeros(4)
        pref = 0.0
        for b in range(a):
            tile = T[4 * a:4 * a + 4, 4 * b:4 * b + 4]
            colT, rowT = tile.sum(axis=0), tile.sum(axis=1)
            for u in range(4):
                F[4 * b + u] += pref + colT[:u].sum()
                rs[u] += rowT[u:].sum()
            pref += tile.sum()
        for x in range(4):
            for y in range(x):
                for u in range(y + 1, x + 1):
                    rs[u] += T[4 * a + x, 4 * a + y]
        F[4 * a:4 * a + 4] += rs
    return F


def test_dlog_alpha_prefix_assembled_from_tiles():
    """The tile decomposition of the pairwise dlog alpha term adds every T_ri
    with i < j <= r exactly once and nothing else: checked on random T, and
    pair by pair with indicator matrices over every pair of the 64-token chunk
    (a missing, doubled or misplaced term shows exactly)."""
    L = 64
    rng = np.random.default_rng(5)
    T = np.tril(rng.standard_normal((L, L)), -1)
    direct = np.array([T[j:, :j].sum() for j in range(L)])
    np.testing.assert_allclose(tile_assembled_F(T), direct, rtol=1e-12, atol=1e-12)
    j = np.arange(L)
    for r in range(L):
        for i in range(r):
            E = np.zeros((L, L))
            E[r, i] = 1.0
            want = ((i < j) & (j <= r)).astype(float)
            np.testing.assert_array_equal(tile_assembled_F(E), want, err_msg=f"pair ({r}, {i})")


def tc_pairwise_terms(kk, qq, g, dAt, dP, L, range_max=80.0):
    """The pairwise gradient stage as the tensor-core kernel forms it, in fp64, for
    one 64-row chunk whose first L rows exist: X1, X2 (row sums) and Y (column sums)
    of the strictly lower dAt and dP as block-referenced products (row block I's
    keys scaled by e^{gb_I - g_i}, gb_I = g at row 16 I - 1 or 0; key block J's rows
    scaled by e^{g_r - ge_J}, ge_J = g at row 16 J + 15; references clamped to the
    last row), blocks spanning more than `range_max` nats summed pairwise, dP's
    diagonal added elementwise, and F(j) = sum_{r >= j} D_r with
    D_r = k_r X1_r + q_r X2_r - k_r Y_r (X2, Y without the diagonal)."""
    C, dk = 64, kk.shape[1]
    kp = np.zeros((C, dk)); kp[:L] = kk[:L]
    qp = np.zeros((C, dk)); qp[:L] = qq[:L]
    gp = np.vstack([g[:L], np.repeat(g[L - 1:L], C - L, axis=0)])
    low = np.tril(np.ones((C, C)), -1)
    A = np.zeros((C, C)); A[:L, :L] = dAt[:L, :L]; A *= low
    Pm = np.zeros((C, C)); Pm[:L, :L] = dP[:L, :L]; Pm *= low
    dPd = np.zeros(C); dPd[:L] = np.diag(dP)[:L]
    ref = [gp[min(16 * j + 15, L - 1)] for j in range(4)]
    gb = [np.zeros(dk)] + ref[:3]
    flag = [np.max(gb[I] - ref[I]) > range_max for I in range(4)]
    X1, X2, Y = np.zeros((C, dk)), np.zeros((C, dk)), np.zeros((C, dk))
    for I in range(4):
        rows, nk = slice(16 * I, 16 * I + 16), 16 * (I + 1)
        KV = kp[:nk] * np.exp(gb[I][None, :] - gp[:nk])
        if flag[I]:
            KV[16 * I:] = 0.0
        sc = np.exp(gp[rows] - gb[I][None, :])
        X1[rows] = (A[rows, :nk] @ KV) * sc
        X2[rows] = (Pm[rows, :nk] @ KV) * sc
    for J in range(4):
        keys, r0 = slice(16 * J, 16 * J + 16), 16 * J
        f = np.exp(gp[r0:] - ref[J][None, :])
        RK, RQ = kp[r0:] * f, qp[r0:] * f
        if flag[J]:
            RK[:16] = 0.0
            RQ[:16] = 0.0
        Y[keys] = (A[r0:, keys].T @ RK + Pm[r0:, keys].T @ RQ) * np.exp(ref[J][None, :] - gp[keys])
    for I in range(4):
        if not flag[I]:
            continue
        for x in range(16 * I + 1, 16 * I + 16):
            for y in range(16 * I, x):
                e = np.exp(gp[x] - gp[y])
                X1[x] += A[x, y] * kp[y] * e
                X2[x] += Pm[x, y] * kp[y] * e
                Y[y] += (A[x, y] * kp[x] + Pm[x, y] * qp[x]) * e
    D = kp * X1 + qp * X2 - kp * Y
    F = np.cumsum(D[::-1], axis=0)[::-1]
    return X1[:L], X2[:L] + dPd[:L, None] * kp[:L], Y[:L] + dPd[:L, None] * qp[:L], F[:L], flag


@pytest.mark.parametrize("L,regime", [(64, "moderate"), (64, "near0"), (50, "mixed")])
def test_tensor_core_pairwise_form_matches_the_pairs(L, regime):
    """The block-referenced form of the pairwise gradient terms (versions and their
    references, the diagonal of dP outside the products, the pairwise path of
    large-range blocks, dlog alpha's pairwise share as a suffix sum of row sums
    minus column sums) equals the direct pairwise sums in fp64.  The near-0 case
    sends every diagonal block down the pairwise path; the mixed case one of them."""
    rng = np.random.default_rng(L + len(regime))
    dk = 8
    kk = rng.standard_normal((L, dk))
    qq = rng.standard_normal((L, dk))
    if regime == "moderate":
        la = -np.logaddexp(0.0, rng.standard_normal((L, dk)) + 2.0)
    elif regime == "near0":
        la = -8.0 - 8.0 * rng.random((L, dk))
    else:
        la = -np.logaddexp(0.0, rng.standard_normal((L, dk)) + 2.0)
        la[16:32] = -8.0 - 8.0 * rng.random((16, dk))
    g = np.cumsum(la, axis=0)
    dAt = rng.standard_normal((L, L))
    dP = rng.standard_normal((L, L))
    X1, X2, Y, F, flag = tc_pairwise_terms(kk, qq, g, dAt, dP, L)
    assert any(flag) == (regime != "moderate")
    E = np.exp(np.minimum(g[:, None, :] - g[None, :, :], 0.0))
    low, inc = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
    A, P = dAt * low, dP * inc
    np.testing.assert_allclose(X1, np.einsum('ri,ic,ric->rc', A, kk, E), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(X2, np.einsum('ri,ic,ric->rc', P, kk, E), rtol=1e-9, atol=1e-12)
    Yd = np.einsum('ri,rc,ric->ic', A, kk, E) + np.einsum('ri,rc,ric->ic', P, qq, E)
    np.testing.assert_allclose(Y, Yd, rtol=1e-9, atol=1e-12)
    Tp = (A[:, :, None] * kk[:, None, :] + P[:, :, None] * qq[:, None, :]) * kk[None, :, :] * E
    Fd = np.array([Tp[j:, :j].sum(axis=(0, 1)) for j in range(L)])
    np.testing.assert_allclose(F, Fd, rtol=1e-8, atol=1e-10)
