"""Pins for the fp64 CPU oracle, against things other than the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong exponent or sign, a transposed operand, an off-by-one in a sweep) fails:

* brute force: the O(T^2) masked sum of the definition, and the matrix forms
  of its three gradients, on tiny inputs with d != e;
* finite differences of L = sum dO * O (O is linear in each single input
  coordinate, so central differences are exact up to rounding);
* a hand-worked example (tests/golden/hand_T3.json);
* closed forms: T = 1, lambda = 1 (textbook masked product), lambda -> 0;
* invariants: causality, linearity in V, homogeneity in Q;
* the tiled algorithm of the pages with the derived decay exponents equals the
  serial recurrence for every tile size, including short last tiles.
"""
import json
import os

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _decay_matrix(T, lam):
    t = np.arange(T)
    lag = t[:, None] - t[None, :]
    D = np.where(lag >= 0, np.power(lam, np.maximum(lag, 0).astype(np.float64)), 0.0)
    return D


def _brute(q, k, v, do, lam):
    """Per-sequence masked products: the definition written as matrices."""
    D = _decay_matrix(q.shape[0], lam)
    A = (q @ k.T) * D            # A_ts = lam^(t-s) (q_t . k_s), s <= t
    G = (do @ v.T) * D           # G_ts = lam^(t-s) (do_t . v_s)
    o = A @ v
    dq = G @ k
    dk = G.T @ q
    dv = A.T @ do
    return o, dq, dk, dv


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


LAMS = [1.0, 0.9, 0.5, 2.0 ** -20]


@pytest.mark.parametrize("T,d,e", [(1, 3, 2), (5, 1, 1), (17, 3, 8), (64, 8, 3)])
def test_brute_force_forward_and_gradients(oracle_mod, T, d, e):
    rng = np.random.default_rng(1234 + T)
    ns = len(LAMS)
    q, k = _rand(rng, ns, T, d), _rand(rng, ns, T, d)
    v, do = _rand(rng, ns, T, e), _rand(rng, ns, T, e)
    lam = np.array(LAMS)
    o = oracle_mod.forward(q, k, v, lam)
    dq, dk, dv = oracle_mod.backward(q, k, v, lam, do)
    for n in range(ns):
        ref = _brute(q[n], k[n], v[n], do[n], lam[n])
        for got, want in zip((o[n], dq[n], dk[n], dv[n]), ref):
            assert _rel(got, want) <= 1e-12


@pytest.mark.parametrize("lam", [1.0, 0.9])
def test_finite_differences(oracle_mod, lam):
    rng = np.random.default_rng(7)
    T, d, e = 6, 3, 2
    q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)

    def loss(qq, kk, vv):
        return float(np.sum(do * oracle_mod.forward(qq[None], kk[None], vv[None], [lam])[0]))

    dq, dk, dv = (g[0] for g in oracle_mod.backward(q[None], k[None], v[None], [lam], do[None]))
    h = 0.5
    for x, g, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        fd = np.zeros_like(x)
        for i in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += h
            xm[i] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            fd[i] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.max(np.abs(fd - g)) <= 1e-10 * max(1.0, np.max(np.abs(g)))


def test_hand_worked_example(oracle_mod):
    with open(os.path.join(GOLDEN, "hand_T3.json")) as f:
        g = json.load(f)
    col = lambda key: np.array(g[key], dtype=np.float64)[None, :, None]
    q, k, v, do = col("q"), col("k"), col("v"), col("do")
    o = oracle_mod.forward(q, k, v, [g["lambda"]])
    dq, dk, dv = oracle_mod.backward(q, k, v, [g["lambda"]], do)
    for key, got in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_array_equal(got[0, :, 0], np.array(g[key]))
    for blk in (1, 2, 3):
        np.testing.assert_array_equal(oracle_mod.forward_blocked(q, k, v, [g["lambda"]], blk)[0, :, 0],
                                      np.array(g["o"]))
        got = oracle_mod.backward_blocked(q, k, v, [g["lambda"]], do, blk)
        for key, x in zip(("dq", "dk", "dv"), got):
            np.testing.assert_array_equal(x[0, :, 0], np.array(g[key]))


def test_T1_closed_form(oracle_mod):
    rng = np.random.default_rng(3)
    d, e = 5, 4
    q, k, v, do = _rand(rng, 3, 1, d), _rand(rng, 3, 1, d), _rand(rng, 3, 1, e), _rand(rng, 3, 1, e)
    lam = np.array([1.0, 0.3, 1e-9])
    o = oracle_mod.forward(q, k, v, lam)
    dq, dk, dv = oracle_mod.backward(q, k, v, lam, do)
    for n in range(3):
        qk = q[n, 0] @ k[n, 0]
        dov = do[n, 0] @ v[n, 0]
        np.testing.assert_allclose(o[n, 0], qk * v[n, 0], rtol=1e-14, atol=0)
        np.testing.assert_allclose(dq[n, 0], dov * k[n, 0], rtol=1e-14, atol=0)
        np.testing.assert_allclose(dk[n, 0], dov * q[n, 0], rtol=1e-14, atol=0)
        np.testing.assert_allclose(dv[n, 0], qk * do[n, 0], rtol=1e-14, atol=0)


def test_lambda_one_is_textbook_causal_linear_attention(oracle_mod):
    rng = np.random.default_rng(11)
    T, d, e = 40, 6, 7
    q, k, v = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e)
    want = np.tril(q @ k.T) @ v
    got = oracle_mod.forward(q[None], k[None], v[None], [1.0])[0]
    assert _rel(got, want) <= 1e-12
    # and, as a prefix sum, o_t = q_t^T sum_{s<=t} k_s v_s^T
    S = np.cumsum(k[:, :, None] * v[:, None, :], axis=0)
    assert _rel(got, np.einsum("td,tde->te", q, S)) <= 1e-12


def test_tiny_lambda_keeps_only_the_diagonal(oracle_mod):
    rng = np.random.default_rng(5)
    T, d, e = 12, 4, 3
    q, k, v = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e)
    lam = 2.0 ** -30
    got = oracle_mod.forward(q[None], k[None], v[None], [lam])[0]
    want = np.sum(q * k, axis=1)[:, None] * v
    assert np.max(np.abs(got - want)) <= 1e-7 * np.max(np.abs(want))


def test_causality(oracle_mod):
    rng = np.random.default_rng(9)
    T, d, e, tp = 30, 4, 5, 17
    q, k, v = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e)
    base = oracle_mod.forward(q[None], k[None], v[None], [0.95])[0]
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[tp:] += 1.0
    k2[tp:] -= 2.0
    v2[tp:] *= 3.0
    pert = oracle_mod.forward(q2[None], k2[None], v2[None], [0.95])[0]
    np.testing.assert_array_equal(pert[:tp], base[:tp])
    assert np.all(np.abs(pert[tp:] - base[tp:]).max(axis=1) > 0)


def test_linearity_and_homogeneity(oracle_mod):
    rng = np.random.default_rng(13)
    T, d, e = 25, 3, 4
    q, k, v1, v2 = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
    f = lambda qq, vv: oracle_mod.forward(qq[None], k[None], vv[None], [0.8])[0]
    assert _rel(f(q, 2.0 * v1 - 3.0 * v2), 2.0 * f(q, v1) - 3.0 * f(q, v2)) <= 1e-12
    assert _rel(f(-1.5 * q, v1), -1.5 * f(q, v1)) <= 1e-12


@pytest.mark.parametrize("T", [1, 7, 64, 65, 129, 300])
@pytest.mark.parametrize("block", [1, 2, 3, 5, 64, 128, 256, "T"])
def test_blocked_equals_serial(oracle_mod, T, block):
    blk = T if block == "T" else block
    rng = np.random.default_rng(T * 1000 + blk)
    d, e = 4, 3
    lam = np.array([1.0, 0.97, 0.5])
    q, k = _rand(rng, 3, T, d), _rand(rng, 3, T, d)
    v, do = _rand(rng, 3, T, e), _rand(rng, 3, T, e)
    o = oracle_mod.forward(q, k, v, lam)
    grads = oracle_mod.backward(q, k, v, lam, do)
    ob = oracle_mod.forward_blocked(q, k, v, lam, blk)
    gb = oracle_mod.backward_blocked(q, k, v, lam, do, blk)
    assert _rel(ob, o) <= 1e-12
    for a, b in zip(gb, grads):
        assert _rel(a, b) <= 1e-12


def test_sequences_are_independent_and_use_their_own_decay(oracle_mod):
    rng = np.random.default_rng(21)
    T, d, e = 20, 3, 2
    q, k, v = _rand(rng, 4, T, d), _rand(rng, 4, T, d), _rand(rng, 4, T, e)
    lam = np.array([0.5, 1.0, 0.9, 0.99])
    together = oracle_mod.forward(q, k, v, lam)
    for n in range(4):
        alone = oracle_mod.forward(q[n:n + 1], k[n:n + 1], v[n:n + 1], lam[n:n + 1])
        np.testing.assert_array_equal(together[n], alone[0])


# ------------------------------------------------------- state in / state out

def _state_closed_form(q, k, v, lam, s0):
    """o_t = lam^(t+1) S0^T q_t + sum_{s<=t} lam^(t-s) (q_t . k_s) v_s and
    S_T = lam^T S0 + sum_s lam^(T-1-s) k_s v_s^T, written out directly."""
    T = q.shape[0]
    D = _decay_matrix(T, lam)
    t = np.arange(T)
    o = ((q @ k.T) * D) @ v + (lam ** (t + 1))[:, None] * (q @ s0)
    w = lam ** (T - 1 - t)
    sT = lam ** T * s0 + (k * w[:, None]).T @ v
    return o, sT


@pytest.mark.parametrize("T,d,e", [(1, 3, 2), (9, 4, 5), (40, 8, 3)])
def test_forward_state_closed_form(oracle_mod, T, d, e):
    rng = np.random.default_rng(77 + T)
    for lam in LAMS:
        q, k, v = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e)
        s0 = _rand(rng, d, e)
        o, sT = oracle_mod.forward_state(q, k, v, lam, s0)
        ro, rs = _state_closed_form(q, k, v, lam, s0)
        assert _rel(o, ro) < 1e-12 and _rel(sT, rs) < 1e-12, lam
        # no initial state: the plain forward, and the state from zero
        o0, s00 = oracle_mod.forward_state(q, k, v, lam)
        ro0, rs0 = _state_closed_form(q, k, v, lam, np.zeros((d, e)))
        assert _rel(o0, ro0) < 1e-12 and _rel(s00, rs0) < 1e-12


@pytest.mark.parametrize("cut", [1, 7, 13, 29])
def test_forward_state_pieces_equal_whole(oracle_mod, cut):
    """Processing [0, cut) and then [cut, T) from the carried state gives the
    outputs and final state of the whole sequence (the state is all that is
    carried)."""
    rng = np.random.default_rng(5 + cut)
    T, d, e = 30, 5, 4
    q, k, v = _rand(rng, 3, T, d), _rand(rng, 3, T, d), _rand(rng, 3, T, e)
    lam = np.array([1.0, 0.9, 0.3])
    o1, s1 = oracle_mod.forward_state(q[:, :cut], k[:, :cut], v[:, :cut], lam)
    o2, s2 = oracle_mod.forward_state(q[:, cut:], k[:, cut:], v[:, cut:], lam, s1)
    o, s = oracle_mod.forward_state(q, k, v, lam)
    assert _rel(np.concatenate([o1, o2], axis=1), o) < 1e-12
    assert _rel(s2, s) < 1e-12


def test_decode_steps_reproduce_the_forward(oracle_mod):
    """T one-token decode steps from a state S0 give the forward's outputs and
    final state from S0."""
    rng = np.random.default_rng(11)
    T, d, e = 12, 4, 6
    q, k, v = _rand(rng, 2, T, d), _rand(rng, 2, T, d), _rand(rng, 2, T, e)
    lam = np.array([0.95, 1.0])
    s0 = _rand(rng, 2, d, e)
    o, sT = oracle_mod.forward_state(q, k, v, lam, s0)
    S = s0.copy()
    outs = []
    for t in range(T):
        ot, S = oracle_mod.decode_step(q[:, t], k[:, t], v[:, t], lam, S)
        outs.append(ot)
    assert _rel(np.stack(outs, axis=1), o) < 1e-12
    assert _rel(S, sT) < 1e-12
    # one step by hand: S' = lam S + k v^T, o = S'^T q
    o1, S1 = oracle_mod.decode_step(q[0, 0], k[0, 0], v[0, 0], lam[0], s0[0])
    Sh = lam[0] * s0[0] + np.outer(k[0, 0], v[0, 0])
    assert _rel(S1, Sh) < 1e-14 and _rel(o1, Sh.T @ q[0, 0]) < 1e-14


# ------------------------------------------------ backward with carried state

def _bwd_state_closed_form(q, k, v, do, lam, s0, g):
    """Gradients of L = sum_t do_t . o_t + <G, S_{T-1}> with S_{-1} = S0,
    written out as matrices:
      dq_t = sum_{s<=t} lam^(t-s) (do_t . v_s) k_s + lam^(t+1) S0 do_t
      dk_s = sum_{t>=s} lam^(t-s) (do_t . v_s) q_t + lam^(T-1-s) G v_s
      dv_s = sum_{t>=s} lam^(t-s) (q_t . k_s) do_t + lam^(T-1-s) G^T k_s
      dS0  = sum_t lam^(t+1) q_t do_t^T + lam^T G
    """
    T = q.shape[0]
    _, dq, dk, dv = _brute(q, k, v, do, lam)
    t = np.arange(T)
    wq = lam ** (t + 1)
    wk = lam ** (T - 1 - t)
    dq = dq + wq[:, None] * (do @ s0.T)
    dk = dk + wk[:, None] * (v @ g.T)
    dv = dv + wk[:, None] * (k @ g)
    ds0 = (q * wq[:, None]).T @ do + lam ** T * g
    return dq, dk, dv, ds0


@pytest.mark.parametrize("T,d,e", [(1, 3, 2), (9, 4, 5), (40, 8, 3)])
def test_backward_state_closed_form(oracle_mod, T, d, e):
    rng = np.random.default_rng(91 + T)
    for lam in LAMS:
        q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
        s0, g = _rand(rng, d, e), _rand(rng, d, e)
        got = oracle_mod.backward_state(q, k, v, lam, do, s0, g)
        want = _bwd_state_closed_form(q, k, v, do, lam, s0, g)
        for a, b in zip(got, want):
            assert _rel(a, b) < 1e-12, lam
        # no states: the plain backward (and dS0 of the plain forward)
        got0 = oracle_mod.backward_state(q, k, v, lam, do)
        want0 = _bwd_state_closed_form(q, k, v, do, lam, np.zeros((d, e)), np.zeros((d, e)))
        for a, b in zip(got0, want0):
            assert _rel(a, b) < 1e-12


@pytest.mark.parametrize("lam", [1.0, 0.9])
def test_backward_state_finite_differences(oracle_mod, lam):
    """Central differences of L = sum do * o + <G, S_T> through forward_state
    (pinned on its own) in every coordinate of S0, q, k and v: L is linear in
    each single coordinate, so the differences are exact up to rounding."""
    rng = np.random.default_rng(8)
    T, d, e = 6, 3, 2
    q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
    s0, g = _rand(rng, d, e), _rand(rng, d, e)

    def loss(qq, kk, vv, ss):
        o, sT = oracle_mod.forward_state(qq, kk, vv, lam, ss)
        return float(np.sum(do * o) + np.sum(g * sT))

    dq, dk, dv, ds0 = oracle_mod.backward_state(q, k, v, lam, do, s0, g)
    h = 0.5
    for arr, grad, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2), (s0, ds0, 3)):
        for pos in np.ndindex(arr.shape):
            args = [q, k, v, s0]
            up, dn = arr.copy(), arr.copy()
            up[pos] += h
            dn[pos] -= h
            args[idx] = up
            lu = loss(*args)
            args[idx] = dn
            ld = loss(*args)
            assert abs((lu - ld) / (2 * h) - grad[pos]) <= 1e-10 * max(1.0, abs(grad[pos]))


@pytest.mark.parametrize("cut", [1, 7, 13, 29])
def test_backward_state_pieces_equal_whole(oracle_mod, cut):
    """A sequence trained in two pieces: the forward of piece 1 gives the state
    S_mid; the backward of piece 2 from S_mid returns dS_mid, which enters the
    backward of piece 1 as the gradient at its final state.  The gradients of
    the pieces, concatenated, and dS0 equal those of the whole sequence."""
    rng = np.random.default_rng(40 + cut)
    T, d, e = 30, 5, 4
    q, k, v, do = (_rand(rng, 3, T, w) for w in (d, d, e, e))
    lam = np.array([1.0, 0.9, 0.3])
    s0, g = _rand(rng, 3, d, e), _rand(rng, 3, d, e)
    _, smid = oracle_mod.forward_state(q[:, :cut], k[:, :cut], v[:, :cut], lam, s0)
    dq2, dk2, dv2, dsmid = oracle_mod.backward_state(q[:, cut:], k[:, cut:], v[:, cut:], lam,
                                                     do[:, cut:], smid, g)
    dq1, dk1, dv1, ds0 = oracle_mod.backward_state(q[:, :cut], k[:, :cut], v[:, :cut], lam,
                                                   do[:, :cut], s0, dsmid)
    whole = oracle_mod.backward_state(q, k, v, lam, do, s0, g)
    for a, b in zip((np.concatenate([dq1, dq2], 1), np.concatenate([dk1, dk2], 1),
                     np.concatenate([dv1, dv2], 1), ds0), whole):
        assert _rel(a, b) < 1e-12


def test_backward_state_empty_sequence(oracle_mod):
    """With no position the final state is S0 itself, so dS0 = G."""
    rng = np.random.default_rng(3)
    d, e = 4, 3
    g = _rand(rng, 2, d, e)
    z = np.zeros((2, 0, d)), np.zeros((2, 0, e))
    out = oracle_mod.backward_state(z[0], z[0], z[1], [0.9, 1.0], z[1], _rand(rng, 2, d, e), g)
    np.testing.assert_array_equal(out[3], g)


# -------------------------------------------------------- gradient in lambda

def _dlambda_closed_form(q, k, v, do, lam, s0, g):
    """dL/dlam for L = sum_t do_t . o_t + <G, S_{T-1}>, written out:
      sum_{s<t} (t-s) lam^(t-s-1) (q_t . k_s)(do_t . v_s)
      + sum_t (t+1) lam^t q_t^T S0 do_t
      + <G, T lam^(T-1) S0 + sum_s (T-1-s) lam^(T-2-s) k_s v_s^T>
    (every power with a zero factor in front taken as 0)."""
    T = q.shape[0]
    t = np.arange(T)
    lag = t[:, None] - t[None, :]
    lagp = np.maximum(lag - 1, 0).astype(np.float64)
    M = np.where(lag >= 1, lag * np.power(lam, lagp), 0.0)
    val = np.sum(M * (q @ k.T) * (do @ v.T))
    val += np.sum((t + 1) * lam ** t * np.einsum("ti,ij,tj->t", q, s0, do))
    w = T - 1 - t
    ws = np.where(w >= 1, w * np.power(lam, np.maximum(w - 1, 0).astype(np.float64)), 0.0)
    dsT = (T * lam ** (T - 1) if T >= 1 else 0.0) * s0 + (k * ws[:, None]).T @ v
    return val + np.sum(g * dsT)


@pytest.mark.parametrize("T,d,e", [(1, 3, 2), (2, 2, 2), (9, 4, 5), (40, 8, 3)])
def test_dlambda_closed_form(oracle_mod, T, d, e):
    rng = np.random.default_rng(300 + T)
    for lam in LAMS:
        q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
        s0, g = _rand(rng, d, e), _rand(rng, d, e)
        got = oracle_mod.dlambda(q, k, v, lam, do, s0, g)
        want = _dlambda_closed_form(q, k, v, do, lam, s0, g)
        assert abs(got - want) <= 1e-11 * max(1.0, abs(want)), (lam, got, want)
        got0 = oracle_mod.dlambda(q, k, v, lam, do)
        want0 = _dlambda_closed_form(q, k, v, do, lam, np.zeros((d, e)), np.zeros((d, e)))
        assert abs(got0 - want0) <= 1e-11 * max(1.0, abs(want0))


@pytest.mark.parametrize("lam", [1.0, 0.9, 0.5])
def test_dlambda_central_differences(oracle_mod, lam):
    """Richardson-extrapolated central differences of L(lam) through
    forward_state (pinned on its own): the step-h and step-h/2 estimates
    combined cancel the h^2 term, leaving O(h^4)."""
    rng = np.random.default_rng(9)
    T, d, e = 7, 3, 2
    q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
    s0, g = _rand(rng, d, e), _rand(rng, d, e)

    def loss(lm):
        o, sT = oracle_mod.forward_state(q, k, v, lm, s0)
        return float(np.sum(do * o) + np.sum(g * sT))

    def cd(h):
        return (loss(lam + h) - loss(lam - h)) / (2 * h)

    h = 1e-3
    est = (4 * cd(h / 2) - cd(h)) / 3
    got = float(oracle_mod.dlambda(q, k, v, lam, do, s0, g))
    assert abs(est - got) <= 1e-8 * max(1.0, abs(got)), (est, got)


def test_dlambda_zero_decay_keeps_lag_one(oracle_mod):
    """At lam = 0 only lag-1 terms survive: sum_t (q_t . k_{t-1})(do_t . v_{t-1})
    + q_0^T S0 do_0 (+ <G, k_{T-2} v_{T-2}^T> from the state)."""
    rng = np.random.default_rng(5)
    T, d, e = 6, 3, 4
    q, k, v, do = _rand(rng, T, d), _rand(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
    s0, g = _rand(rng, d, e), _rand(rng, d, e)
    want = sum(float(q[t] @ k[t - 1]) * float(do[t] @ v[t - 1]) for t in range(1, T))
    want += float(q[0] @ s0 @ do[0]) + float(np.sum(g * np.outer(k[T - 2], v[T - 2])))
    got = float(oracle_mod.dlambda(q, k, v, 0.0, do, s0, g))
    assert abs(got - want) <= 1e-12 * max(1.0, abs(want))


# ------------------------------------------------------ normalised variant

def _norm_closed_form(q, k, v, dy, lam):
    """The normalised form and its gradients as matrices, D_ts = lam^(t-s) [s<=t]:
      num = ((Q K^T) * D) V,  z = D K,  den = rowsum(Q * z),  y = num / den
      dnum = dy / den,  dden = -rowsum(dy * num) / den^2
      dQ = ((dnum V^T) * D) K + dden z
      dK = ((dnum V^T) * D)^T Q + D^T (dden Q)
      dV = ((Q K^T) * D)^T dnum"""
    D = _decay_matrix(q.shape[0], lam)
    A = (q @ k.T) * D
    num = A @ v
    z = D @ k
    den = np.sum(q * z, axis=1)
    y = num / den[:, None]
    dnum = dy / den[:, None]
    dden = -np.sum(dy * num, axis=1) / den ** 2
    G = (dnum @ v.T) * D
    dq1, dq2 = G @ k, dden[:, None] * z
    dk1, dk2 = G.T @ q, D.T @ (dden[:, None] * q)
    dv = A.T @ dnum
    # the two parts of dq (and of dk) cancel where y hardly depends on q (k),
    # e.g. T = 1 or a tiny decay; compare those against the parts' size
    scale = (None, None, max(np.max(np.abs(dq1)), np.max(np.abs(dq2))),
             max(np.max(np.abs(dk1)), np.max(np.abs(dk2))), None)
    return (y, den, dq1 + dq2, dk1 + dk2, dv), scale


def _positive(rng, *shape):
    return np.abs(rng.standard_normal(shape)) + 0.1


@pytest.mark.parametrize("T,d,e", [(1, 3, 2), (9, 4, 5), (40, 8, 3)])
def test_norm_closed_form(oracle_mod, T, d, e):
    rng = np.random.default_rng(500 + T)
    for lam in LAMS:
        q, k = _positive(rng, T, d), _positive(rng, T, d)
        v, dy = _rand(rng, T, e), _rand(rng, T, e)
        y, den = oracle_mod.forward_norm(q, k, v, lam)
        grads = oracle_mod.backward_norm(q, k, v, lam, dy)
        want, scale = _norm_closed_form(q, k, v, dy, lam)
        for a, b, sc in zip((y, den) + tuple(grads), want, scale):
            ref = np.max(np.abs(b)) if sc is None else max(sc, np.max(np.abs(b)))
            assert np.max(np.abs(a - b)) <= 1e-12 * ref, lam


def test_norm_single_position_returns_v(oracle_mod):
    """T = 1: y = (q.k) v / (q.k) = v whatever q and k, so dq = dk = 0, dv = dy."""
    rng = np.random.default_rng(2)
    q, k, v, dy = _positive(rng, 1, 4), _positive(rng, 1, 4), _rand(rng, 1, 3), _rand(rng, 1, 3)
    y, _ = oracle_mod.forward_norm(q, k, v, 0.7)
    dq, dk, dv = oracle_mod.backward_norm(q, k, v, 0.7, dy)
    assert _rel(y, v) < 1e-15 and np.max(np.abs(dq)) < 1e-15 and np.max(np.abs(dk)) < 1e-15
    assert _rel(dv, dy) < 1e-15


def test_norm_scale_invariance(oracle_mod):
    """y does not change when q or k is scaled by a positive constant."""
    rng = np.random.default_rng(3)
    q, k, v = _positive(rng, 2, 20, 4), _positive(rng, 2, 20, 4), _rand(rng, 2, 20, 3)
    lam = np.array([0.9, 1.0])
    y, _ = oracle_mod.forward_norm(q, k, v, lam)
    assert _rel(oracle_mod.forward_norm(3.0 * q, k, v, lam)[0], y) < 1e-13
    assert _rel(oracle_mod.forward_norm(q, 0.25 * k, v, lam)[0], y) < 1e-13


def test_norm_central_differences(oracle_mod):
    """Richardson-extrapolated central differences of L = sum dy * y in every
    coordinate of q, k and v (y is not linear in q or k, so plain differences
    would carry an h^2 error)."""
    rng = np.random.default_rng(4)
    T, d, e, lam = 5, 3, 2, 0.9
    q, k, v, dy = _positive(rng, T, d), _positive(rng, T, d), _rand(rng, T, e), _rand(rng, T, e)
    grads = oracle_mod.backward_norm(q, k, v, lam, dy)

    def loss(args):
        return float(np.sum(dy * oracle_mod.forward_norm(*args, lam)[0]))

    for idx, (arr, g) in enumerate(zip((q, k, v), grads)):
        for pos in np.ndindex(arr.shape):
            def cd(h):
                args = [q, k, v]
                up, dn = arr.copy(), arr.copy()
                up[pos] += h
                dn[pos] -= h
                args[idx] = up
                lu = loss(args)
                args[idx] = dn
                return (lu - loss(args)) / (2 * h)
            est = (4 * cd(1e-3) - cd(2e-3)) / 3
            assert abs(est - g[pos]) <= 1e-8 * max(1.0, abs(g[pos])), (idx, pos, est, g[pos])
