"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test names the page and section it rests on.  Page shorthands:
  essay   -- "From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252
  explain -- "我终于看懂了 KDA" explainer, pwwt.cn/news/3787313
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 1234


def _rand_inputs(n_tok, H, dk, dv, seed, alpha_mode="channel", beta_mode="rand"):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_tok, H, dk))
    k = rng.standard_normal((n_tok, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((n_tok, H, dv))
    if alpha_mode == "channel":
        la = -np.log1p(np.exp(rng.standard_normal((n_tok, H, dk)) + 1.0))
    elif alpha_mode == "scalar":
        la = np.repeat(-np.log1p(np.exp(rng.standard_normal((n_tok, H, 1)) + 1.0)), dk, axis=-1)
    elif alpha_mode == "one":
        la = np.zeros((n_tok, H, dk))
    elif alpha_mode == "zero":
        la = np.full((n_tok, H, dk), -np.inf)
    else:
        raise ValueError(alpha_mode)
    if beta_mode == "rand":
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((n_tok, H))))
    elif beta_mode == "one":
        beta = np.ones((n_tok, H))
    else:
        beta = np.zeros((n_tok, H))
    return q, k, v, la, beta


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b ** 2)), 1e-300)


# ---------------------------------------------------------------- golden cases

def test_hand_worked_two_tokens():
    """Two steps worked by hand (tests/golden/hand_two_tokens.json); order of
    operations from explain s8, learning rate from explain s6, per-channel
    alpha from explain s9."""
    g = json.load(open(os.path.join(GOLDEN, "hand_two_tokens.json")))
    q = np.array(g["q"])[:, None, :]
    k = np.array(g["k"])[:, None, :]
    v = np.array(g["v"])[:, None, :]
    la = np.log(np.array(g["alpha"]))[:, None, :]
    beta = np.array(g["beta"])[:, None]
    o, fs = oracle.forward(q, k, v, la, beta, [0, 2])
    np.testing.assert_allclose(o[:, 0, :], np.array(g["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], np.array(g["final_state"]), rtol=0, atol=1e-14)
    for C in (1, 2):
        out = oracle.chunkform(q, k, v, la, beta, [0, 2], C)
        np.testing.assert_allclose(out["o"][:, 0, :], np.array(g["o"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(out["final_state"][0, 0], np.array(g["final_state"]), rtol=0, atol=1e-14)


def test_status_board_overwrite():
    """explain s1 / s6: the board keeps only the latest status per key; the delta
    rule (essay) with beta = alpha = 1 replaces the old value exactly."""
    g = json.load(open(os.path.join(GOLDEN, "status_board.json")))
    k = np.array(g["k"], dtype=float)[:, None, :]
    q = np.array(g["q"], dtype=float)[:, None, :]
    v = np.array(g["v"], dtype=float)[:, None, :]
    n = k.shape[0]
    la = np.zeros_like(k)
    beta = np.ones((n, 1))
    o, fs = oracle.forward(q, k, v, la, beta, [0, n])
    np.testing.assert_array_equal(o[:, 0, :], np.array(g["o"]))
    np.testing.assert_array_equal(fs[0, 0], np.array(g["final_state"]))
    for C in (1, 2, 3, 5, 8):
        out = oracle.chunkform(q, k, v, la, beta, [0, n], C)
        np.testing.assert_allclose(out["o"][:, 0, :], np.array(g["o"]), atol=1e-14)


# ---------------------------------------------------------------- special cases

def test_P1_alpha_one_is_deltanet():
    """essay, delta rule: M <- M + beta (v - M k) k^T with M = S^T (d_v x d_k, the
    page's orientation); alpha = 1 must give exactly this."""
    q, k, v, la, beta = _rand_inputs(40, 2, 5, 3, 1, alpha_mode="one")
    o, fs = oracle.forward(q, k, v, la, beta, [0, 40])
    for h in range(2):
        M = np.zeros((3, 5))
        for t in range(40):
            M = M + beta[t, h] * np.outer(v[t, h] - M @ k[t, h], k[t, h])
            np.testing.assert_allclose(o[t, h], M @ q[t, h], atol=1e-12)
        np.testing.assert_allclose(fs[0, h], M.T, atol=1e-12)


def test_P2_scalar_alpha_is_gated_deltanet():
    """essay, Gated DeltaNet: one alpha per head; a scalar commutes with the
    projector, so S <- alpha (I - beta k k^T) S + beta k v^T."""
    q, k, v, la, beta = _rand_inputs(30, 2, 4, 3, 2, alpha_mode="scalar")
    o, fs = oracle.forward(q, k, v, la, beta, [0, 30])
    for h in range(2):
        S = np.zeros((4, 3))
        for t in range(30):
            a = np.exp(la[t, h, 0])
            S = a * (np.eye(4) - beta[t, h] * np.outer(k[t, h], k[t, h])) @ S + beta[t, h] * np.outer(k[t, h], v[t, h])
            np.testing.assert_allclose(o[t, h], S.T @ q[t, h], atol=1e-12)
        np.testing.assert_allclose(fs[0, h], S, atol=1e-12)


def test_P3_alpha_zero_clears_memory():
    """essay, Gated DeltaNet: alpha = 0 clears the memory, so o_t depends on token
    t only: o_t = beta_t (q_t . k_t) v_t and S_T = beta_T k_T v_T^T, whatever S_0."""
    q, k, v, la, beta = _rand_inputs(17, 3, 6, 4, 3, alpha_mode="zero")
    s0 = np.random.default_rng(9).standard_normal((1, 3, 6, 4))
    for init in (None, s0):
        o, fs = oracle.forward(q, k, v, la, beta, [0, 17], init_state=init)
        expect = beta[:, :, None] * np.sum(q * k, axis=-1)[:, :, None] * v
        np.testing.assert_allclose(o, expect, atol=1e-14)
        np.testing.assert_allclose(fs[0], beta[-1][:, None, None] * k[-1][:, :, None] * v[-1][:, None, :],
                                   atol=1e-14)
        for C in (1, 4, 16, 17):
            out = oracle.chunkform(q, k, v, la, beta, [0, 17], C, init_state=init)
            np.testing.assert_allclose(out["o"], expect, atol=1e-13)


def test_P4_orthonormal_keys_exact_retrieval():
    """explain s1 / s6: with beta = 1, alpha = 1 and orthonormal keys, querying
    with a key returns the last value written under it."""
    rng = np.random.default_rng(4)
    dk, dv, T = 6, 5, 40
    basis, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    idx = rng.integers(0, dk, size=T)
    qidx = rng.integers(0, dk, size=T)
    k = basis.T[idx][:, None, :]
    q = basis.T[qidx][:, None, :]
    v = rng.standard_normal((T, 1, dv))
    la = np.zeros((T, 1, dk))
    beta = np.ones((T, 1))
    o, fs = oracle.forward(q, k, v, la, beta, [0, T])
    last = {}
    for t in range(T):
        last[idx[t]] = v[t, 0]
        expect = last.get(qidx[t], np.zeros(dv))
        np.testing.assert_allclose(o[t, 0], expect, atol=1e-12)
    for C in (1, 7, 16, 40):
        out = oracle.chunkform(q, k, v, la, beta, [0, T], C)
        np.testing.assert_allclose(out["o"], o, atol=1e-12)


def test_P4b_identical_keys_overwrite():
    """explain s11: two writes under the same key -- the second overwrites the first."""
    k1 = np.array([0.6, 0.0, 0.8])
    k = np.stack([k1, k1])[:, None, :]
    q = k.copy()
    v = np.array([[1.0, 2.0], [-3.0, 0.5]])[:, None, :]
    la = np.zeros((2, 1, 3))
    beta = np.ones((2, 1))
    o, _ = oracle.forward(q, k, v, la, beta, [0, 2])
    np.testing.assert_allclose(o[1, 0], v[1, 0], atol=1e-15)


def test_P5_beta_zero_alpha_one_passes_state():
    """explain s6: a zero learning rate writes nothing; alpha = 1 decays nothing:
    S_T = S_0 and o_t = S_0^T q_t."""
    q, k, v, la, beta = _rand_inputs(20, 2, 4, 3, 5, alpha_mode="one", beta_mode="zero")
    s0 = np.random.default_rng(6).standard_normal((1, 2, 4, 3))
    o, fs = oracle.forward(q, k, v, la, beta, [0, 20], init_state=s0)
    np.testing.assert_array_equal(fs, s0)
    np.testing.assert_allclose(o, np.einsum("thc,hcj->thj", q, s0[0]), atol=1e-14)


def test_P8_beta_zero_is_pure_decay():
    """explain s8 / s10: with no writes the state only decays, channel by channel:
    S_T[c,:] = (prod_t alpha_t[c]) S_0[c,:]; the norm never grows."""
    q, k, v, la, beta = _rand_inputs(25, 2, 4, 3, 7, beta_mode="zero")
    s0 = np.random.default_rng(8).standard_normal((1, 2, 4, 3))
    norms = []
    for T in range(1, 26):
        _, fs = oracle.forward(q[:T], k[:T], v[:T], la[:T], beta[:T], [0, T], init_state=s0)
        norms.append(np.linalg.norm(fs))
    assert all(b <= a + 1e-15 for a, b in zip(norms, norms[1:]))
    expect = np.exp(la.sum(axis=0))[:, :, None] * s0[0]
    np.testing.assert_allclose(fs[0], expect, rtol=1e-12)


def test_P7_update_is_gradient_step():
    """Online-gradient-descent reading of the delta rule (engineer's blog,
    cnnetsun.cn/a/3598456; explain s7): the write equals -beta * grad_S of
    0.5 * ||S^T k - v||^2 at the decayed state, checked by finite differences."""
    q, k, v, la, beta = _rand_inputs(1, 1, 4, 3, 11)
    s0 = np.random.default_rng(12).standard_normal((1, 1, 4, 3))
    _, fs = oracle.forward(q, k, v, la, beta, [0, 1], init_state=s0)
    Sd = np.exp(la[0, 0])[:, None] * s0[0, 0]
    loss = lambda S: 0.5 * np.sum((S.T @ k[0, 0] - v[0, 0]) ** 2)
    grad = np.zeros_like(Sd)
    eps = 1e-6
    for c in range(4):
        for j in range(3):
            E = np.zeros_like(Sd)
            E[c, j] = eps
            grad[c, j] = (loss(Sd + E) - loss(Sd - E)) / (2 * eps)
    np.testing.assert_allclose(fs[0, 0] - Sd, -beta[0, 0] * grad, atol=1e-8)


def test_P9_dense_transition_product():
    """North-star matrix form, as a product of dense d_k x d_k transitions:
    S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, tiny sizes."""
    q, k, v, la, beta = _rand_inputs(8, 2, 3, 2, 13)
    s0 = np.random.default_rng(14).standard_normal((1, 2, 3, 2))
    o, fs = oracle.forward(q, k, v, la, beta, [0, 8], init_state=s0)
    for h in range(2):
        # S_T = Phi_{T..1} S_0 + sum_t Phi_{T..t+1} beta_t k_t v_t^T
        Ms = [(np.eye(3) - beta[t, h] * np.outer(k[t, h], k[t, h])) @ np.diag(np.exp(la[t, h])) for t in range(8)]
        for T in range(1, 9):
            Phi = np.eye(3)
            for t in range(T):
                Phi = Ms[t] @ Phi
            S = Phi @ s0[0, h]
            for t in range(T):
                P = np.eye(3)
                for u in range(t + 1, T):
                    P = Ms[u] @ P
                S = S + P @ (beta[t, h] * np.outer(k[t, h], v[t, h]))
            np.testing.assert_allclose(o[T - 1, h], S.T @ q[T - 1, h], atol=1e-12)
        np.testing.assert_allclose(fs[0, h], S, atol=1e-12)


def test_linear_in_state_and_values():
    """Structural fact of the matrix form: (o, S_T) is linear in (S_0, V) jointly."""
    q, k, v, la, beta = _rand_inputs(19, 2, 5, 4, 15)
    s0 = np.random.default_rng(16).standard_normal((1, 2, 5, 4))
    o1, f1 = oracle.forward(q, k, v, la, beta, [0, 19], init_state=s0)
    o2, f2 = oracle.forward(q, k, np.zeros_like(v), la, beta, [0, 19], init_state=s0)
    o3, f3 = oracle.forward(q, k, v, la, beta, [0, 19], init_state=None)
    np.testing.assert_allclose(o1, o2 + o3, atol=1e-12)
    np.testing.assert_allclose(f1, f2 + f3, atol=1e-12)


# ---------------------------------------------------------------- chunk form

@pytest.mark.parametrize("C", [1, 3, 16, 64, 128, 1000])
def test_P6_chunk_size_independence(C):
    """essay, chunkwise paragraph: the chunk size changes the schedule, not the
    result; C = 1 is the token recurrence, C >= length is one masked block."""
    lens = [37, 130, 1, 64, 0, 200]
    seq = np.concatenate([[0], np.cumsum(lens)])
    n = int(seq[-1])
    q, k, v, la, beta = _rand_inputs(n, 2, 8, 6, 21)
    la[5:9, 0, :3] = -np.inf                      # some alpha = 0 channels
    la[50, 1, :] = -np.inf
    s0 = np.random.default_rng(22).standard_normal((len(lens), 2, 8, 6)) * 0.3
    o, fs = oracle.forward(q, k, v, la, beta, seq, init_state=s0)
    out = oracle.chunkform(q, k, v, la, beta, seq, C, init_state=s0)
    assert _rel(out["o"], o) < 1e-10
    assert _rel(out["final_state"], fs) < 1e-10


def test_chunk_intermediates_against_recurrence():
    """The chunk-form intermediates, checked against the token recurrence:
    * the start state of chunk n equals the recurrence's state after n*C tokens;
    * W row r is the rank-one write of token r: S_r - Diag(alpha_r) S_{r-1} = k_r W_r^T;
    * U = W at zero start state, and W is affine in S_0 with slope -Wk
      (perturbing S_0[c, j] moves column j of W by -Wk[:, c]);
    * g is the chunk-restarting running sum of log alpha."""
    C, T, H, dk, dv = 8, 21, 1, 4, 3
    q, k, v, la, beta = _rand_inputs(T, H, dk, dv, 31)
    s0 = np.random.default_rng(32).standard_normal((1, H, dk, dv))
    seq = [0, T]
    out = oracle.chunkform(q, k, v, la, beta, seq, C, init_state=s0, intermediates=True)
    states = [s0[0, 0]]
    for t in range(1, T + 1):
        _, fs = oracle.forward(q[:t], k[:t], v[:t], la[:t], beta[:t], [0, t], init_state=s0)
        states.append(fs[0, 0])
    for n in range(3):
        np.testing.assert_allclose(out["s_chunk"][n, 0], states[n * C], atol=1e-12)
    for t in range(T):
        write = states[t + 1] - np.exp(la[t, 0])[:, None] * states[t]
        np.testing.assert_allclose(write, np.outer(k[t, 0], out["w"][t, 0]), atol=1e-12)
    # U and Wk from the affine dependence of W on the chunk start state (first chunk)
    out0 = oracle.chunkform(q, k, v, la, beta, seq, C, init_state=np.zeros_like(s0), intermediates=True)
    np.testing.assert_allclose(out0["u"][:C], out0["w"][:C], atol=1e-12)
    np.testing.assert_allclose(out["u"][:C], out0["u"][:C], atol=1e-12)
    for c in range(dk):
        for j in range(dv):
            E = np.zeros_like(s0)
            E[0, 0, c, j] = 1.0
            oute = oracle.chunkform(q, k, v, la, beta, seq, C, init_state=E, intermediates=True)
            np.testing.assert_allclose(oute["w"][:C, 0, j] - out0["w"][:C, 0, j], -out0["wk"][:C, 0, c],
                                       atol=1e-12)
    for n0 in range(0, T, C):
        np.testing.assert_allclose(out["g"][n0:n0 + C], np.cumsum(la[n0:n0 + C], axis=0), atol=1e-12)


def test_decode_step_is_one_token():
    """explain s15: decode reads the state, emits the output, updates the state;
    N sequences with one token each."""
    q, k, v, la, beta = _rand_inputs(5, 2, 4, 3, 41)
    s0 = np.random.default_rng(42).standard_normal((5, 2, 4, 3))
    o, s1 = oracle.decode_step(q, k, v, la, beta, s0)
    for n in range(5):
        o_n, f_n = oracle.forward(q[n:n + 1], k[n:n + 1], v[n:n + 1], la[n:n + 1], beta[n:n + 1], [0, 1],
                                  init_state=s0[n:n + 1])
        np.testing.assert_array_equal(o[n], o_n[0])
        np.testing.assert_array_equal(s1[n], f_n[0])


# ---------------------------------------------------------- input preprocessing
# tahou -- "22580倍参数量级" article, tahou.com/article/213680821660188677
# (alpha between 0 and 1 from an "alpha projection"; alpha = 1 is the delta
# rule, alpha = 0 clears the memory).  The -softplus / sigmoid / L2-norm maps
# are this library's reading of how raw projections reach those ranges.

from oracle import prep  # noqa: E402


def test_l2_normalize_closed_forms():
    np.testing.assert_allclose(prep.l2_normalize([3.0, 4.0]), [0.6, 0.8], rtol=0, atol=1e-15)
    np.testing.assert_allclose(prep.l2_normalize([[0.0, -2.0, 0.0]]), [[0.0, -1.0, 0.0]], atol=0)
    x = np.random.default_rng(3).standard_normal((4, 3, 7))
    x[1, 2] = 0.0                                           # all-zero row stays zero, no NaN
    y = prep.l2_normalize(x)
    n = np.linalg.norm(y, axis=-1)
    np.testing.assert_allclose(np.delete(n.reshape(-1), 5), 1.0, atol=1e-14)   # over the last axis
    assert np.all(y[1, 2] == 0.0)
    np.testing.assert_allclose(np.linalg.norm(x, axis=-1, keepdims=True) * y, x, atol=1e-14)
    c = np.random.default_rng(4).uniform(0.1, 10.0, size=(4, 3, 1))
    np.testing.assert_allclose(prep.l2_normalize(c * x), y, atol=1e-14)       # positive scale invariance
    np.testing.assert_allclose(prep.l2_normalize(-x), -y, atol=0)


def test_gate_softplus_closed_forms():
    ln3 = np.log(3.0)
    np.testing.assert_allclose(prep.log_alpha_from_gate([0.0, ln3, -ln3]),
                               [-np.log(2.0), -np.log(4.0), -np.log(4.0 / 3.0)], rtol=1e-15)
    np.testing.assert_allclose(np.exp(prep.log_alpha_from_gate(ln3)), 0.25, rtol=1e-15)   # alpha = 1/(1+3)
    a = np.random.default_rng(5).standard_normal(1000) * 6.0
    la = prep.log_alpha_from_gate(a)
    assert np.all(la < 0.0)                                                # alpha in (0, 1)
    np.testing.assert_allclose(prep.log_alpha_from_gate(-a) - la, a, atol=1e-12)   # sp(x) - sp(-x) = x
    np.testing.assert_allclose(prep.log_alpha_from_gate(50.0), -50.0, rtol=1e-15)
    np.testing.assert_allclose(prep.log_alpha_from_gate(-50.0), -np.exp(-50.0), rtol=1e-12)
    assert prep.log_alpha_from_gate(-800.0) == 0.0                         # alpha = 1: delta rule
    assert np.exp(prep.log_alpha_from_gate(800.0)) == 0.0                  # alpha = 0: clear
    h = 1e-5                                                               # d/da softplus = sigmoid
    d = -(prep.log_alpha_from_gate(a + h) - prep.log_alpha_from_gate(a - h)) / (2 * h)
    np.testing.assert_allclose(d, prep.beta_from_logit(a), atol=1e-9)


def test_beta_sigmoid_closed_forms():
    ln3 = np.log(3.0)
    np.testing.assert_allclose(prep.beta_from_logit([0.0, ln3, -ln3]), [0.5, 0.75, 0.25], rtol=1e-15)
    b = np.random.default_rng(6).standard_normal(1000) * 8.0
    s = prep.beta_from_logit(b)
    assert np.all((s > 0.0) & (s < 1.0))
    np.testing.assert_allclose(s + prep.beta_from_logit(-b), 1.0, atol=1e-15)
    assert prep.beta_from_logit(-1000.0) == 0.0 and prep.beta_from_logit(1000.0) == 1.0
    assert np.all(np.diff(prep.beta_from_logit(np.sort(b))) >= 0.0)       # increasing


def test_preprocess_flags_select_their_inputs():
    rng = np.random.default_rng(7)
    q, k, g = (rng.standard_normal((5, 2, 4)) * 3 for _ in range(3))
    b = rng.standard_normal((5, 2))
    for flags in range(8):
        q2, k2, g2, b2 = prep.preprocess(q, k, g, b, flags)
        same = lambda x, y: np.array_equal(x, y)
        assert same(q2, q) != bool(flags & prep.QK_L2NORM)
        assert same(k2, k) != bool(flags & prep.QK_L2NORM)
        assert same(g2, g) != bool(flags & prep.GATE_SOFTPLUS)
        assert same(b2, b) != bool(flags & prep.BETA_SIGMOID)
        if flags & prep.QK_L2NORM:
            np.testing.assert_allclose(np.linalg.norm(k2, axis=-1), 1.0, atol=1e-14)
            np.testing.assert_allclose(np.linalg.norm(q2, axis=-1), 1.0, atol=1e-14)


def test_prep_forward_scale_invariance_and_gate_limits():
    """With the L2 norm, rescaling any token's raw q or k by a positive number
    changes nothing; gate logits of -800 / +800 give the delta rule / a cleared
    memory (tahou, Gated DeltaNet section)."""
    rng = np.random.default_rng(8)
    T, H, dk, dv = 19, 2, 6, 5
    q, k, g = (rng.standard_normal((T, H, dk)) for _ in range(3))
    v = rng.standard_normal((T, H, dv))
    b = rng.standard_normal((T, H))
    s0 = rng.standard_normal((1, H, dk, dv))
    allf = prep.QK_L2NORM | prep.GATE_SOFTPLUS | prep.BETA_SIGMOID
    o1, f1 = oracle.forward(*_order(prep.preprocess(q, k, g, b, allf), v), [0, T], init_state=s0)
    cq, ck = rng.uniform(0.05, 20.0, (T, H, 1)), rng.uniform(0.05, 20.0, (T, H, 1))
    o2, f2 = oracle.forward(*_order(prep.preprocess(cq * q, ck * k, g, b, allf), v), [0, T], init_state=s0)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(f2, f1, atol=1e-12)
    # all logits -800: alpha = 1 exactly, the delta rule (log alpha = 0)
    qn, kn, la0, bn = prep.preprocess(q, k, np.full_like(g, -800.0), b, allf)
    assert np.all(la0 == 0.0)
    # token 7 with logits +800: alpha = 0, the memory before it is cleared
    gc = g.copy()
    gc[7] = 800.0
    oc, fc = oracle.forward(*_order(prep.preprocess(q, k, gc, b, allf), v), [0, T], init_state=s0)
    qn, kn, la, bn = prep.preprocess(q, k, gc, b, allf)
    of, ff = oracle.forward(qn[7:], kn[7:], v[7:], la[7:], bn[7:], [0, T - 7], init_state=np.zeros_like(s0))
    np.testing.assert_allclose(oc[7:], of, atol=1e-12)
    np.testing.assert_allclose(fc, ff, atol=1e-12)


def _order(pre, v):
    q, k, la, b = pre
    return q, k, v, la, b


# ------------------------------------------------------------- backward (O3)
# The pages give no backward derivation (training is only said to need the
# parallel form); O3 is pinned to the forward oracle, which is pinned above, by
# finite differences and by exact identities of the recurrence.

def _loss_inputs(seed, lens=(5, 0, 4), H=2, dk=3, dv=2):
    seq = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq[-1])
    q, k, v, la, beta = _rand_inputs(T, H, dk, dv, seed)
    rng = np.random.default_rng(seed + 1)
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    do = rng.standard_normal((T, H, dv))
    dfs = rng.standard_normal((len(lens), H, dk, dv))
    return seq, q, k, v, la, beta, s0, do, dfs


def _loss(seq, q, k, v, la, beta, s0, do, dfs):
    o, fs = oracle.forward(q, k, v, la, beta, seq, init_state=s0)
    return float(np.sum(o * do) + np.sum(fs * dfs))


def test_backward_matches_central_differences():
    """Every gradient entry (q, k, v, log alpha, beta, initial state) against a
    central difference of the fp64 forward; sequences of length 5, 0 and 4."""
    seq, q, k, v, la, beta, s0, do, dfs = _loss_inputs(51)
    g = oracle.backward(q, k, v, la, beta, seq, do, d_final_state=dfs, init_state=s0)
    args = {"q": q, "k": k, "v": v, "la": la, "beta": beta, "s0": s0}
    names = {"q": "dq", "k": "dk", "v": "dv", "la": "dlog_alpha", "beta": "dbeta", "s0": "d_init_state"}
    h = 1e-6
    for name, x in args.items():
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = _loss(seq, args["q"], args["k"], args["v"], args["la"], args["beta"], args["s0"], do, dfs)
            x[idx] = old - h
            lm = _loss(seq, args["q"], args["k"], args["v"], args["la"], args["beta"], args["s0"], do, dfs)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[names[name]], fd, atol=2e-7, rtol=1e-6, err_msg=name)


def test_backward_homogeneity_identities():
    """o and the final state are jointly linear in (V, S0), and o is linear in
    q (the final state does not depend on q), so by Euler's identity
    <dV, V> + <dS0, S0> = L and <dq, q> = <do, o> exactly (up to rounding)."""
    seq, q, k, v, la, beta, s0, do, dfs = _loss_inputs(52, lens=(37, 1, 70), H=3, dk=8, dv=5)
    g = oracle.backward(q, k, v, la, beta, seq, do, d_final_state=dfs, init_state=s0)
    o, fs = oracle.forward(q, k, v, la, beta, seq, init_state=s0)
    L = np.sum(o * do) + np.sum(fs * dfs)
    np.testing.assert_allclose(np.sum(g["dv"] * v) + np.sum(g["d_init_state"] * s0), L, rtol=1e-10)
    np.testing.assert_allclose(np.sum(g["dq"] * q), np.sum(o * do), rtol=1e-10)


def test_backward_alpha_zero_cuts_the_gradient():
    """alpha = 0 at token 40 clears the memory (tahou, Gated DeltaNet section):
    outputs from token 40 on do not depend on anything before it, so changing
    their upstream gradients leaves the gradients of tokens 0..39 and of S0
    unchanged, and log alpha at token 40 gets zero gradient (the decayed state
    is zero)."""
    seq, q, k, v, la, beta, s0, do, dfs = _loss_inputs(53, lens=(90,), H=2, dk=6, dv=4)
    la[40] = -np.inf
    g1 = oracle.backward(q, k, v, la, beta, seq, do, d_final_state=dfs, init_state=s0)
    do2 = do.copy()
    do2[40:] = np.random.default_rng(9).standard_normal(do2[40:].shape)
    g2 = oracle.backward(q, k, v, la, beta, seq, do2, d_final_state=2 * dfs, init_state=s0)
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        np.testing.assert_array_equal(g1[name][:40], g2[name][:40], err_msg=name)
    np.testing.assert_array_equal(g1["d_init_state"], g2["d_init_state"])
    assert np.all(g1["dlog_alpha"][40] == 0.0)
    assert not np.allclose(g1["dv"][40:], g2["dv"][40:])


def test_backward_long_sequence_crosses_checkpoints():
    """A 200-token sequence (checkpoint copies every 64 tokens) gives the same
    gradients as the same tokens run as one forward/backward with the state
    handed over at token 130 (two sequences chained through the initial
    state and its gradient)."""
    seq, q, k, v, la, beta, s0, do, dfs = _loss_inputs(54, lens=(200,), H=1, dk=5, dv=3)
    g = oracle.backward(q, k, v, la, beta, seq, do, d_final_state=dfs, init_state=s0)
    a, b = slice(0, 130), slice(130, 200)
    _, s_mid = oracle.forward(q[a], k[a], v[a], la[a], beta[a], [0, 130], init_state=s0)
    g2 = oracle.backward(q[b], k[b], v[b], la[b], beta[b], [0, 70], do[b], d_final_state=dfs, init_state=s_mid)
    g1 = oracle.backward(q[a], k[a], v[a], la[a], beta[a], [0, 130], do[a], d_final_state=g2["d_init_state"],
                         init_state=s0)
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        np.testing.assert_allclose(np.concatenate([g1[name], g2[name]]), g[name], rtol=1e-9, atol=1e-12,
                                   err_msg=name)
    np.testing.assert_allclose(g1["d_init_state"], g["d_init_state"], rtol=1e-9, atol=1e-12)
