"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-worked example, a closed form, an invariant, a limiting case the pages
state, an independently written formulation, or brute force with explicit
matrices.  ``test_oracle_mutants.py`` plants mistakes in a copy of the oracle
and checks that these pins catch every one.
"""
import json
import os

import numpy as np
import pytest

from conftest import rel_l2_per_slice

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand_problem(rng, T, hk, hv, dk, dv, s0=True, unit_keys=True, g_scale=1.0):
    q = rng.standard_normal((1, T, hk, dk))
    k = rng.standard_normal((1, T, hk, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, hv, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, hv))))
    g = -g_scale * np.logaddexp(0.0, rng.standard_normal((1, T, hv)))
    S0 = 0.3 * rng.standard_normal((1, hv, dv, dk)) if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------------------
# Hand-worked example (pencil and paper; tests/golden/handworked_d2.json)
# ---------------------------------------------------------------------------
def test_handworked_example(oracle_mod):
    with open(os.path.join(HERE, "golden", "handworked_d2.json")) as f:
        gold = json.load(f)
    q = np.array(gold["q"])[None, :, None, :]
    k = np.array(gold["k"])[None, :, None, :]
    v = np.array(gold["v"])[None, :, None, :]
    beta = np.array(gold["beta"])[None, :, None]
    g = np.array(gold["g"])[None, :, None]
    o, sf = oracle_mod.recurrent(q, k, v, g, beta)
    np.testing.assert_allclose(o[0, :, 0, :], np.array(gold["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf[0, 0], np.array(gold["s_final"]), rtol=0, atol=1e-12)
    for C in (1, 2, 3):
        oc, sc = oracle_mod.chunkwise(q, k, v, g, beta, C)
        np.testing.assert_allclose(oc[0, :, 0, :], np.array(gold["o"]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(sc[0, 0], np.array(gold["s_final"]), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# P-6: one token from a zero state: o = beta v (k.q), S = beta v k^T, and the
# grouped-head mapping (value head h reads q/k head h // (Hv/Hk)).
# ---------------------------------------------------------------------------
def test_one_token_and_head_mapping(oracle_mod):
    rng = np.random.default_rng(6)
    hk, hv, dk, dv = 2, 6, 5, 3
    q, k, v, g, beta, _ = _rand_problem(rng, 1, hk, hv, dk, dv, s0=False)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta)
    for h in range(hv):
        hq = h // (hv // hk)
        kq = k[0, 0, hq] @ q[0, 0, hq]
        np.testing.assert_allclose(o[0, 0, h], beta[0, 0, h] * v[0, 0, h] * kq, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(sf[0, h], beta[0, 0, h] * np.outer(v[0, 0, h], k[0, 0, hq]), rtol=1e-13,
                                   atol=1e-15)


# ---------------------------------------------------------------------------
# P-2: g = 0 (alpha = 1) is DeltaNet; compare with the error-correcting form
# S <- S - beta (S k - v) k^T, written separately.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("s0", [False, True])
def test_g_zero_is_delta_rule(oracle_mod, s0):
    rng = np.random.default_rng(2)
    q, k, v, g, beta, S0 = _rand_problem(rng, 40, 2, 4, 8, 6, s0=s0)
    g = np.zeros_like(g)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    od, sd = oracle_mod.delta_error_form(q, k, v, beta, initial_state=S0)
    assert rel_l2_per_slice(o[0], od[0], axes=(0, 2)) < 1e-13
    assert rel_l2_per_slice(sf, sd, axes=(2, 3)) < 1e-13


# ---------------------------------------------------------------------------
# P-3: beta = 0 leaves only the decay: S_t = exp(g_1 + ... + g_t) S0 and
# o_t = exp(G_t) S0 q_t.  With g = 0 as well, S is unchanged.
# ---------------------------------------------------------------------------
def test_beta_zero_decay_only(oracle_mod):
    rng = np.random.default_rng(3)
    hk, hv, dk, dv, T = 1, 2, 6, 4, 17
    q, k, v, g, beta, S0 = _rand_problem(rng, T, hk, hv, dk, dv)
    beta = np.zeros_like(beta)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    G = np.cumsum(g[0], axis=0)  # [T, hv]
    for h in range(hv):
        np.testing.assert_allclose(sf[0, h], np.exp(G[-1, h]) * S0[0, h], rtol=1e-13)
        for t in range(T):
            np.testing.assert_allclose(o[0, t, h], np.exp(G[t, h]) * S0[0, h] @ q[0, t, 0], rtol=1e-12,
                                       atol=1e-300)
    o2, sf2 = oracle_mod.recurrent(q, k, v, np.zeros_like(g), beta, initial_state=S0)
    np.testing.assert_array_equal(sf2, S0)
    for t in range(T):
        np.testing.assert_allclose(o2[0, t, 0], S0[0, 0] @ q[0, t, 0], rtol=1e-13)


# ---------------------------------------------------------------------------
# P-4: exact recall.  alpha = 1, beta = 1, orthonormal keys written in order:
# S k_i = v_i for every written pair, S = S0 (I - sum k k^T) + sum v k^T.
# ---------------------------------------------------------------------------
def test_exact_recall_orthonormal_keys(oracle_mod):
    rng = np.random.default_rng(4)
    d, m, dv = 8, 6, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:, :m].T  # m orthonormal rows
    k = keys[None, :, None, :]
    q = rng.standard_normal((1, m, 1, d))
    v = rng.standard_normal((1, m, 1, dv))
    beta = np.ones((1, m, 1))
    g = np.zeros((1, m, 1))
    S0 = rng.standard_normal((1, 1, dv, d))
    _, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    S = sf[0, 0]
    for i in range(m):
        np.testing.assert_allclose(S @ keys[i], v[0, i, 0], rtol=1e-12, atol=1e-12)
    P = keys.T @ keys
    np.testing.assert_allclose(S, S0[0, 0] @ (np.eye(d) - P) + v[0, :, 0].T @ keys, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# P-5: alpha -> 0 (g = -inf) clears the state: S_t = beta v k^T and
# o_t = beta v (k.q), whatever came before.
# ---------------------------------------------------------------------------
def test_alpha_zero_clears_state(oracle_mod):
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = _rand_problem(rng, 9, 1, 2, 4, 3)
    g[:] = -np.inf
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    for h in range(2):
        for t in range(9):
            np.testing.assert_allclose(o[0, t, h], beta[0, t, h] * v[0, t, h] * (k[0, t, 0] @ q[0, t, 0]),
                                       rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(sf[0, h], beta[0, -1, h] * np.outer(v[0, -1, h], k[0, -1, 0]), rtol=1e-13)


# ---------------------------------------------------------------------------
# P-7: the norm bound that unit keys and beta in (0,1) give:
# ||S_t||_2 <= alpha_t ||S_{t-1}||_2 + beta_t ||v_t|| ||k_t||.
# ---------------------------------------------------------------------------
def test_norm_bound(oracle_mod):
    rng = np.random.default_rng(7)
    T, dk, dv = 60, 6, 5
    q, k, v, g, beta, S0 = _rand_problem(rng, T, 1, 1, dk, dv, g_scale=0.05)
    S = S0[0, 0]
    for t in range(T):
        sl = slice(t, t + 1)
        _, sf = oracle_mod.recurrent(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl],
                                     initial_state=S[None, None])
        Sn = sf[0, 0]
        bound = np.exp(g[0, t, 0]) * np.linalg.norm(S, 2) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0]) * \
            np.linalg.norm(k[0, t, 0])
        assert np.linalg.norm(Sn, 2) <= bound * (1 + 1e-12)
        # the transition alone is a contraction along k: ||S(I - beta k k^T)|| <= ||S||
        M = np.eye(dk) - beta[0, t, 0] * np.outer(k[0, t, 0], k[0, t, 0])
        assert np.linalg.norm(M, 2) <= 1 + 1e-12
        S = Sn


# ---------------------------------------------------------------------------
# P-9: brute force with explicit d x d matrices of the pages' product form:
# S_T = S0 prod_t M_t + sum_s beta_s v_s k_s^T prod_{t>s} M_t,
# M_t = alpha_t (I - beta_t k_t k_t^T);  o_t = S_t q_t.
# ---------------------------------------------------------------------------
def test_brute_force_explicit_matrices(oracle_mod):
    rng = np.random.default_rng(9)
    T, hk, hv, dk, dv = 7, 1, 2, 5, 3
    q, k, v, g, beta, S0 = _rand_problem(rng, T, hk, hv, dk, dv, unit_keys=False)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    for h in range(hv):
        Ms = [np.exp(g[0, t, h]) * (np.eye(dk) - beta[0, t, h] * np.outer(k[0, t, 0], k[0, t, 0])) for t in range(T)]
        for tt in range(T):
            P = np.eye(dk)
            for t in range(tt + 1):
                P = P @ Ms[t]
            St = S0[0, h] @ P
            for s in range(tt + 1):
                R = np.eye(dk)
                for t in range(s + 1, tt + 1):
                    R = R @ Ms[t]
                St = St + beta[0, s, h] * np.outer(v[0, s, h], k[0, s, 0]) @ R
            np.testing.assert_allclose(o[0, tt, h], St @ q[0, tt, 0], rtol=1e-11, atol=1e-13)
            if tt == T - 1:
                np.testing.assert_allclose(sf[0, h], St, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------------------
# P-1: the chunkwise (WY/UT) form equals the recurrence to 1e-12 -- several
# chunk sizes, grouped heads, d_k != d_v, varlen with ragged tails.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 4, 16])
@pytest.mark.parametrize("s0", [False, True])
def test_chunkwise_equals_recurrent(oracle_mod, C, s0):
    rng = np.random.default_rng(11 + C)
    lens = [37, 1, 16, 64, 5]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta, _ = _rand_problem(rng, T, 2, 4, 12, 10)
    S0 = 0.3 * rng.standard_normal((len(lens), 4, 10, 12)) if s0 else None
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0, cu_seqlens=cu)
    oc, sc = oracle_mod.chunkwise(q, k, v, g, beta, C, initial_state=S0, cu_seqlens=cu)
    assert rel_l2_per_slice(oc, o, axes=(0, 2)) < 1e-12
    assert rel_l2_per_slice(sc, sf, axes=(2, 3)) < 1e-12


def test_chunkwise_strong_decay_and_clearing(oracle_mod):
    """Very negative g (exp(g) underflows to exactly 0 in fp64) keeps the chunk
    form finite: Gamma is built as exp(G_r - G_j), never as a ratio of
    underflowed products.  (g = -inf itself is a limit of the recurrence,
    pinned by test_alpha_zero_clears_state; prefix sums of -inf are not
    defined, so the chunk form takes finite g.)"""
    rng = np.random.default_rng(12)
    q, k, v, g, beta, S0 = _rand_problem(rng, 48, 1, 1, 6, 6)
    g[0, ::7, 0] = -200.0
    g[0, 5, 0] = -1000.0
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    oc, sc = oracle_mod.chunkwise(q, k, v, g, beta, 16, initial_state=S0)
    assert np.all(np.isfinite(oc)) and np.all(np.isfinite(sc))
    assert rel_l2_per_slice(oc, o, axes=(1, 3)) < 1e-12
    assert rel_l2_per_slice(sc, sf, axes=(2, 3)) < 1e-12


# ---------------------------------------------------------------------------
# Chunk intermediates pinned to per-token quantities.  The state at each
# chunk start must equal the recurrence run up to that token; the rows of
# U are u_r = beta_r (v_r - alpha_r S_{r-1} k_r); U is affine in S0 with
# U(S0=0) = U~ and U(0) - U(S0) = W S0^T.
# ---------------------------------------------------------------------------
def test_chunk_intermediates_pinned_by_recurrence(oracle_mod):
    rng = np.random.default_rng(13)
    C, T, dk, dv = 8, 29, 6, 5
    q, k, v, g, beta, S0 = _rand_problem(rng, T, 1, 1, dk, dv)
    _, _, inter = oracle_mod.chunkwise(q, k, v, g, beta, C, initial_state=S0, intermediates=True)
    _, _, inter0 = oracle_mod.chunkwise(q, k, v, g, beta, C, initial_state=None, intermediates=True)
    # per-token states by running the recurrence on every prefix
    states = [S0[0, 0]]
    for t in range(T):
        _, sf = oracle_mod.recurrent(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], g[:, :t + 1], beta[:, :t + 1],
                                     initial_state=S0)
        states.append(sf[0, 0])
    for c, c0 in enumerate(range(0, T, C)):
        np.testing.assert_allclose(inter["sc"][c, 0], states[c0], rtol=1e-12, atol=1e-13)
        L = min(C, T - c0)
        for r in range(L):
            t = c0 + r
            u_ref = beta[0, t, 0] * (v[0, t, 0] - np.exp(g[0, t, 0]) * states[t] @ k[0, t, 0])
            np.testing.assert_allclose(inter["u"][c, 0, r], u_ref, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(inter["gcum"][c, 0, r], g[0, c0:t + 1, 0].sum(), rtol=1e-13)
        # U~ is U with a zero start state only for the first chunk (later
        # chunks start from the carried state), so compare affine parts
        if c == 0:
            np.testing.assert_allclose(inter0["u"][c, 0, :L], inter["ut"][c, 0, :L], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(inter0["u"][c, 0, :L] - inter["u"][c, 0, :L],
                                       inter["w"][c, 0, :L] @ S0[0, 0].T, rtol=1e-11, atol=1e-13)
        # T is unit lower-triangular
        Tm = inter["tmat"][c, 0, :L, :L]
        np.testing.assert_array_equal(np.diag(Tm), np.ones(L))
        assert np.all(np.triu(Tm, 1) == 0)


# ---------------------------------------------------------------------------
# P-8: continuation.  run(x[:T1]) -> S; run(x[T1:], S) equals run(x); and
# one-token decode steps after a prefill equal a longer prefill.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T1", [1, 13, 31])
def test_continuation(oracle_mod, T1):
    rng = np.random.default_rng(8)
    T = 32
    q, k, v, g, beta, S0 = _rand_problem(rng, T, 2, 4, 7, 5)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    a = slice(0, T1)
    b = slice(T1, T)
    oa, sa = oracle_mod.recurrent(q[:, a], k[:, a], v[:, a], g[:, a], beta[:, a], initial_state=S0)
    ob, sb = oracle_mod.recurrent(q[:, b], k[:, b], v[:, b], g[:, b], beta[:, b], initial_state=sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sb, sf, rtol=1e-12, atol=1e-14)
    # decode steps after the prefix
    S = sa
    for t in range(T1, T):
        od, S = oracle_mod.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        np.testing.assert_allclose(od[0], o[0, t], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S, sf, rtol=1e-12, atol=1e-14)


def test_varlen_equals_per_sequence(oracle_mod):
    rng = np.random.default_rng(10)
    lens = [3, 0, 11, 1]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta, _ = _rand_problem(rng, T, 1, 2, 4, 4)
    S0 = rng.standard_normal((len(lens), 2, 4, 4))
    o, sf = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        if L == 0:
            np.testing.assert_array_equal(sf[n], S0[n])  # empty sequence: final = initial
            continue
        on, sn = oracle_mod.recurrent(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], initial_state=S0[n:n + 1])
        np.testing.assert_array_equal(o[0, cu[n]:cu[n + 1]], on[0])
        np.testing.assert_array_equal(sf[n], sn[0])


def test_unit_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(14)
    q, k, v, g, beta, _ = _rand_problem(rng, 20, 2, 4, 5, 5)
    q = np.concatenate([q, q[:, ::-1]], axis=0)
    k = np.concatenate([k, k], axis=0)
    v = np.concatenate([v, v], axis=0)
    g = np.concatenate([g, g], axis=0)
    beta = np.concatenate([beta, beta], axis=0)
    o, sf = oracle_mod.recurrent(q, k, v, g, beta)
    units = [1, 6]
    os_, ss = oracle_mod.recurrent(q, k, v, g, beta, units=units)
    for u in units:
        n, h = divmod(u, 4)
        np.testing.assert_array_equal(os_[n, :, h], o[n, :, h])
        np.testing.assert_array_equal(ss[n, h], sf[n, h])
    assert np.isnan(os_[0, :, 0]).all()


def test_prepare_closed_forms(oracle_mod):
    """The input side: log-sigmoid and sigmoid closed forms, and the
    invariants of per-head L2 normalisation."""
    rng = np.random.default_rng(40)
    q = rng.standard_normal((7, 3, 8))
    k = 5.0 * rng.standard_normal((7, 3, 8))
    k[2, 1] = 0.0  # a zero row stays zero (the 1e-12 floor of the norm)
    a = np.tile(np.array([0.0, 40.0, -40.0, 1.5, -3.0, 0.25]), (7, 1))
    b = -a
    q2, k2, g2, b2 = oracle_mod.prepare_inputs(q, k, a, b, qk_l2norm=True, gate_logits=True)
    assert np.allclose(np.linalg.norm(q2, axis=-1), 1.0, atol=1e-15)
    assert np.allclose(np.sum(q2 * q, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-14)
    assert np.all(k2[2, 1] == 0.0)
    kn = np.linalg.norm(k, axis=-1)
    ok = kn > 0
    assert np.allclose(np.linalg.norm(k2, axis=-1)[ok], 1.0, atol=1e-15)
    # log sigmoid: g(0) = -ln 2; g(40) = -e^-40 to first order; g(-40) = -40 in fp64
    assert abs(g2[0, 0] + np.log(2.0)) < 1e-16
    assert abs(g2[0, 1] + np.exp(-40.0)) < 1e-33
    assert g2[0, 2] == -40.0
    # e^{log sigmoid(a)} + sigmoid(-a) = 1 ties the two gates together; sigmoid(0) = 1/2
    assert np.allclose(np.exp(g2) + b2, 1.0, atol=2e-16)
    assert b2[0, 0] == 0.5
    # a positive scale of the raw projections does not change the normalised rows
    q3, k3, _, _ = oracle_mod.prepare_inputs(3.7 * q, 0.01 * k, a, b, qk_l2norm=True)
    assert np.allclose(q3, q2, atol=1e-15) and np.allclose(k3[ok], k2[ok], atol=1e-15)
    # flags off: values unchanged
    q4, k4, g4, b4 = oracle_mod.prepare_inputs(q, k, a, b)
    assert np.array_equal(q4, q) and np.array_equal(k4, k) and np.array_equal(g4, a) and np.array_equal(b4, b)


def test_prepared_one_token_closed_form(oracle_mod):
    """From a zero state, one token of raw inputs gives
    o = sigmoid(b) v (k . q) / (|k| |q|), whatever the decay logit."""
    rng = np.random.default_rng(41)
    d, hk, hv = 6, 1, 2
    q = rng.standard_normal((1, 1, hk, d))
    k = 3.0 * rng.standard_normal((1, 1, hk, d))
    v = rng.standard_normal((1, 1, hv, d))
    a = rng.standard_normal((1, 1, hv))
    b = rng.standard_normal((1, 1, hv))
    q2, k2, g2, b2 = oracle_mod.prepare_inputs(q, k, a, b, qk_l2norm=True, gate_logits=True)
    o, sf = oracle_mod.recurrent(q2, k2, v, g2, b2)
    cosine = float(np.dot(q[0, 0, 0], k[0, 0, 0]) / (np.linalg.norm(q[0, 0, 0]) * np.linalg.norm(k[0, 0, 0])))
    for h in range(hv):
        sig = 1.0 / (1.0 + np.exp(-b[0, 0, h]))
        assert np.allclose(o[0, 0, h], sig * cosine * v[0, 0, h], rtol=1e-13, atol=1e-15)
        assert np.allclose(sf[0, h], sig * np.outer(v[0, 0, h], k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])),
                           rtol=1e-13, atol=1e-15)


def test_output_side_handworked(oracle_mod):
    """The output side on a two-channel row worked by hand: o = (3, 4) has
    mean square 12.5, so the normalised row is (3, 4) / sqrt(12.5) =
    (0.8485..., 1.1313...); sigmoid(ln 3) = 3/4, so SiLU(ln 3) = (3/4) ln 3;
    SiLU(0) = 0 and sigmoid(0) = 1/2."""
    o = np.array([[[3.0, 4.0]]])
    r = np.sqrt(12.5)
    y = oracle_mod.output_side(o, eps=0.0)
    assert np.allclose(y, [[[3.0 / r, 4.0 / r]]], rtol=1e-15)
    w = np.array([2.0, 0.5])
    z = np.array([[[0.0, np.log(3.0)]]])
    y = oracle_mod.output_side(o, z=z, weight=w, eps=0.0, gate="silu")
    assert np.allclose(y, [[[0.0, 2.0 / r * 0.75 * np.log(3.0)]]], rtol=1e-15, atol=0)
    y = oracle_mod.output_side(o, z=z, weight=w, eps=0.0, gate="sigmoid")
    assert np.allclose(y, [[[0.5 * 6.0 / r, 0.75 * 2.0 / r]]], rtol=1e-15)
    # eps inside the root: a constant row c gives c / sqrt(c^2 + eps)
    c = np.full((1, 1, 5), 0.2)
    y = oracle_mod.output_side(c, eps=0.01)
    assert np.allclose(y, 0.2 / np.sqrt(0.04 + 0.01), rtol=1e-15)


def test_output_side_invariants(oracle_mod):
    """Invariants of RMS normalisation on random rows: mean(y^2) =
    ms / (ms + eps) with unit scale; a positive rescaling of o leaves y
    unchanged when eps = 0; the zero-centred scale 1 + w equals the plain
    scale 1 + w; per-head scales act on their own head only."""
    rng = np.random.default_rng(42)
    T, hv, dv = 6, 3, 16
    o = rng.standard_normal((T, hv, dv)) * rng.uniform(0.2, 3.0, (T, hv, 1))
    ms = np.mean(o * o, axis=-1)
    eps = 0.3
    y = oracle_mod.output_side(o, eps=eps)
    assert np.allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-14)
    assert np.allclose(oracle_mod.output_side(7.5 * o, eps=0.0), oracle_mod.output_side(o, eps=0.0), rtol=1e-14)
    d = 0.1 * rng.standard_normal(dv)
    assert np.allclose(oracle_mod.output_side(o, weight=d, eps=eps, zero_centred=True),
                       oracle_mod.output_side(o, weight=1.0 + d, eps=eps), rtol=1e-15)
    assert np.array_equal(oracle_mod.output_side(o, eps=eps, zero_centred=True), y)
    wh = np.stack([np.full(dv, h + 1.0) for h in range(hv)])
    yh = oracle_mod.output_side(o, weight=wh, eps=eps)
    for h in range(hv):
        assert np.allclose(yh[:, h], (h + 1.0) * y[:, h], rtol=1e-15)
    # the gate multiplies elementwise: SiLU(z) = z sigmoid(z), against numpy
    z = rng.standard_normal((T, hv, dv)) * 3.0
    yg = oracle_mod.output_side(o, z=z, eps=eps, gate="silu")
    assert np.allclose(yg, y * z / (1.0 + np.exp(-z)), rtol=1e-14)


def _kda_problem(rng, T, hk, hv, d, s0=True, g_scale=1.0):
    q, k, v, g, beta, S0 = _rand_problem(rng, T, hk, hv, d, d, s0=s0)
    gk = -g_scale * np.logaddexp(0.0, rng.standard_normal((1, T, hv, d)))
    return q, k, v, gk, beta, S0


def test_kda_scalar_decay_is_gated_delta_rule(oracle_mod):
    """KDA with the same decay on every key channel is the gated delta rule
    ("Gated Attention Architectures", section 8: KDA reduces to Gated
    DeltaNet when the decay collapses to a scalar per head)."""
    rng = np.random.default_rng(50)
    q, k, v, g, beta, S0 = _rand_problem(rng, 41, 2, 4, 8, 8)
    gk = np.repeat(g[..., None], 8, axis=-1)
    o1, s1 = oracle_mod.kda_recurrent(q, k, v, gk, beta, initial_state=S0)
    o2, s2 = oracle_mod.recurrent(q, k, v, g, beta, initial_state=S0)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13) and np.allclose(s1, s2, rtol=1e-12, atol=1e-13)


def test_kda_brute_force_explicit_matrices(oracle_mod):
    """KDA against explicit d x d transition matrices: with M_t =
    diag(alpha_t)(I - beta_t k_t k_t^T) (this build's orientation, the
    transpose of the page's (I - beta k k^T) D_t), S_t = S_{t-1} M_t +
    beta_t v_t k_t^T and o_t = S_t q_t, multiplied out token by token."""
    rng = np.random.default_rng(51)
    T, d = 9, 5
    q, k, v, gk, beta, S0 = _kda_problem(rng, T, 1, 1, d)
    o, sf = oracle_mod.kda_recurrent(q, k, v, gk, beta, initial_state=S0)
    S = S0[0, 0].copy()
    for t in range(T):
        kt, qt, vt, bt = k[0, t, 0], q[0, t, 0], v[0, t, 0], beta[0, t, 0]
        M = np.diag(np.exp(gk[0, t, 0])) @ (np.eye(d) - bt * np.outer(kt, kt))
        S = S @ M + bt * np.outer(vt, kt)
        assert np.allclose(o[0, t, 0], S @ qt, rtol=1e-12, atol=1e-13)
    assert np.allclose(sf[0, 0], S, rtol=1e-12, atol=1e-13)


def test_kda_beta_zero_is_channel_decay(oracle_mod):
    """beta = 0: only the decay acts, per key channel: S_T = S_0 diag(e^{sum g})
    and o_t = S_0 (e^{G_t} .* q_t)."""
    rng = np.random.default_rng(52)
    q, k, v, gk, beta, S0 = _kda_problem(rng, 12, 1, 2, 6)
    beta = np.zeros_like(beta)
    o, sf = oracle_mod.kda_recurrent(q, k, v, gk, beta, initial_state=S0)
    G = np.cumsum(gk[0], axis=0)  # [T, hv, d]
    for h in range(2):
        assert np.allclose(sf[0, h], S0[0, h] * np.exp(G[-1, h])[None, :], rtol=1e-13)
        for t in range(12):
            assert np.allclose(o[0, t, h], S0[0, h] @ (np.exp(G[t, h]) * q[0, t, 0]), rtol=1e-12, atol=1e-14)


def test_kda_one_token(oracle_mod):
    """One token from a start state S: o = S D q + beta (v - S D k)(k . q)
    with D = diag(alpha); from zero, o = beta v (k . q) whatever the decay."""
    rng = np.random.default_rng(53)
    q, k, v, gk, beta, S0 = _kda_problem(rng, 1, 1, 1, 7)
    D = np.exp(gk[0, 0, 0])
    S, kt, qt, vt, bt = S0[0, 0], k[0, 0, 0], q[0, 0, 0], v[0, 0, 0], beta[0, 0, 0]
    o, _ = oracle_mod.kda_recurrent(q, k, v, gk, beta, initial_state=S0)
    ref = S @ (D * qt) + bt * (vt - S @ (D * kt)) * (kt @ qt)
    assert np.allclose(o[0, 0, 0], ref, rtol=1e-13)
    o0, _ = oracle_mod.kda_recurrent(q, k, v, gk, beta)
    assert np.allclose(o0[0, 0, 0], bt * vt * (kt @ qt), rtol=1e-13)


@pytest.mark.parametrize("C", [1, 4, 16])
def test_kda_chunkwise_equals_recurrent(oracle_mod, C):
    """The KDA chunked form (derived separately, masked products formed term
    by term) against the token recurrence, batched and packed, with start
    states and strong per-channel decay."""
    rng = np.random.default_rng(54)
    q, k, v, gk, beta, S0 = _kda_problem(rng, 45, 2, 4, 8, g_scale=3.0)
    o1, s1 = oracle_mod.kda_recurrent(q, k, v, gk, beta, initial_state=S0)
    o2, s2 = oracle_mod.kda_chunkwise(q, k, v, gk, beta, C, initial_state=S0)
    assert np.allclose(o1, o2, rtol=1e-11, atol=1e-13) and np.allclose(s1, s2, rtol=1e-11, atol=1e-13)
    lens = [0, 7, 17, 21]
    cu = np.concatenate([[0], np.cumsum(lens)])
    s0v = 0.3 * rng.standard_normal((4, 4, 8, 8))
    o3, s3 = oracle_mod.kda_recurrent(q[0], k[0], v[0], gk[0], beta[0], initial_state=s0v, cu_seqlens=cu)
    o4, s4 = oracle_mod.kda_chunkwise(q[0], k[0], v[0], gk[0], beta[0], C, initial_state=s0v, cu_seqlens=cu)
    assert np.allclose(o3, o4, rtol=1e-11, atol=1e-13) and np.allclose(s3, s4, rtol=1e-11, atol=1e-13)
    assert np.array_equal(s3[0], s0v[0])  # the empty sequence keeps its state


def _fd_grads(oracle_mod, args, dO, dSf, names, h=1e-6, cu=None):
    """Central finite differences of L = sum dO . o + sum dSf . S_T through the
    (pinned) forward recurrence."""
    def loss(a):
        o, sf = oracle_mod.recurrent(a["q"], a["k"], a["v"], a["g"], a["beta"], initial_state=a["s0"], cu_seqlens=cu)
        return float((o * dO).sum() + (sf * dSf).sum())
    out = {}
    for name in names:
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            ap, am = dict(args), dict(args)
            ap[name] = x.copy()
            am[name] = x.copy()
            ap[name][idx] += h
            am[name][idx] -= h
            fd[idx] = (loss(ap) - loss(am)) / (2 * h)
        out[name] = fd
    return out


def test_backward_matches_finite_differences(oracle_mod):
    """Every gradient of the hand-written reverse recurrence against central
    differences of the forward recurrence (grouped heads, a start state,
    unnormalised keys)."""
    rng = np.random.default_rng(60)
    T, hk, hv, d = 7, 1, 2, 3
    q, k, v, g, beta, S0 = _rand_problem(rng, T, hk, hv, d, d, unit_keys=False)
    k *= 0.6
    dO = rng.standard_normal(v.shape)
    dSf = rng.standard_normal(S0.shape)
    gr = oracle_mod.backward(q, k, v, g, beta, dO, dSf, initial_state=S0)
    args = dict(q=q, k=k, v=v, g=g, beta=beta, s0=S0)
    fd = _fd_grads(oracle_mod, args, dO, dSf, list(args))
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"), ("s0", "dS0")):
        ref = fd[name]
        got = gr[key].reshape(ref.shape)
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-7), (name, np.abs(got - ref).max())


def test_backward_varlen_finite_differences(oracle_mod):
    """Packed sequences (one empty): gradients stay inside their sequence and
    an empty sequence passes dS_final straight to dS0."""
    rng = np.random.default_rng(61)
    lens = [3, 0, 4]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, hk, hv, d = sum(lens), 1, 1, 3
    q, k, v, g, beta, _ = _rand_problem(rng, T, hk, hv, d, d, s0=False)
    q, k, v, g, beta = q[0], k[0], v[0], g[0], beta[0]
    S0 = 0.3 * rng.standard_normal((3, hv, d, d))
    dO = rng.standard_normal(v.shape)
    dSf = rng.standard_normal(S0.shape)
    gr = oracle_mod.backward(q, k, v, g, beta, dO, dSf, initial_state=S0, cu_seqlens=cu)
    args = dict(q=q, k=k, v=v, g=g, beta=beta, s0=S0)
    fd = _fd_grads(oracle_mod, args, dO, dSf, ["k", "g", "s0"], cu=cu)
    assert np.allclose(gr["dk"], fd["k"], rtol=1e-6, atol=1e-7)
    assert np.allclose(gr["dg"], fd["g"], rtol=1e-6, atol=1e-7)
    assert np.allclose(gr["dS0"], fd["s0"], rtol=1e-6, atol=1e-7)
    assert np.array_equal(gr["dS0"][1], dSf[1])


@pytest.mark.parametrize("C", [1, 4, 16])
def test_backward_chunkwise_equals_token_recurrence(oracle_mod, C):
    """The chunked form differentiated (matrix calculus through the WY
    inverse and the decay masks) against the token recurrence's reverse
    mode: two derivations of the same gradients."""
    rng = np.random.default_rng(62)
    q, k, v, g, beta, S0 = _rand_problem(rng, 37, 2, 4, 8, 8, g_scale=2.0)
    dO = rng.standard_normal(v.shape)
    dSf = rng.standard_normal(S0.shape)
    a = oracle_mod.backward(q, k, v, g, beta, dO, dSf, initial_state=S0)
    b = oracle_mod.backward(q, k, v, g, beta, dO, dSf, initial_state=S0, chunk=C)
    for n in a:
        assert np.allclose(a[n], b[n], rtol=1e-10, atol=1e-11), (n, np.abs(a[n] - b[n]).max())


# ---------------------------------------------------------------------------
# The input side's short causal convolution ("Architecture Thread I",
# "Modern Architecture Improvements": projection -> short conv -> SiLU)
# ---------------------------------------------------------------------------

def _conv_case(rng, lens, channels=(2, 3), W=4):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x = rng.standard_normal((sum(lens), *channels))
    w = rng.standard_normal((*channels, W))
    st = rng.standard_normal((len(lens), *channels, W - 1))
    return cu, x, w, st


def test_short_conv_identity_and_shift(oracle_mod):
    """The last tap is the current token: a kernel (0, .., 0, 1) is the
    identity; (1, 0, .., 0) delays by W - 1 tokens, reading the conv state
    (or zeros) before the sequence's first token."""
    rng = np.random.default_rng(70)
    W = 4
    cu, x, _, st = _conv_case(rng, [6, 2], channels=(3,), W=W)
    ident = np.zeros((3, W))
    ident[:, -1] = 1.0
    y, s = oracle_mod.short_conv(x, ident, cu_seqlens=cu, state=st, silu=False)
    assert np.array_equal(y, x)
    delay = np.zeros((3, W))
    delay[:, 0] = 1.0
    y, s = oracle_mod.short_conv(x, delay, cu_seqlens=cu, silu=False)
    assert np.array_equal(y[:3], np.zeros((3, 3))) and np.array_equal(y[3:6], x[0:3])
    assert np.array_equal(y[6:8], np.zeros((2, 3)))  # the second sequence never sees the first
    y, s = oracle_mod.short_conv(x, delay, cu_seqlens=cu, state=st, silu=False)
    assert np.array_equal(y[0:3], st[0].T) and np.array_equal(y[6:8], st[1].T[0:2])
    # the state after a sequence: its last W - 1 inputs, oldest first; the 2-token sequence keeps
    # the newest entry of its incoming state in front of its two inputs
    assert np.array_equal(s[0], x[3:6].T)
    assert np.array_equal(s[1][:, 0], st[1][:, -1]) and np.array_equal(s[1][:, 1:], x[6:8].T)


def test_short_conv_equals_numpy_correlate(oracle_mod):
    """Against numpy's correlation of (state, sequence) with each channel's
    filter, and SiLU against scipy's logistic: packed sequences of lengths
    0 to 9, W = 1, 2 and 4."""
    from scipy.special import expit
    rng = np.random.default_rng(71)
    for W in (1, 2, 4):
        lens = [5, 0, 1, 9, 2]
        cu, x, w, st = _conv_case(rng, lens, W=W)
        y, s = oracle_mod.short_conv(x, w, cu_seqlens=cu, state=st, silu=False)
        ys, _ = oracle_mod.short_conv(x, w, cu_seqlens=cu, state=st, silu=True)
        for n in range(len(lens)):
            a, b = cu[n], cu[n + 1]
            for c0 in range(2):
                for c1 in range(3):
                    full = np.concatenate([st[n, c0, c1], x[a:b, c0, c1]])
                    if b > a:
                        ref = np.correlate(full, w[c0, c1], mode="valid")
                        assert np.allclose(y[a:b, c0, c1], ref, rtol=1e-13, atol=1e-13)
                    assert np.allclose(s[n, c0, c1], full[len(full) - (W - 1):], rtol=0, atol=0)
        assert np.allclose(ys, y * expit(y), rtol=1e-13, atol=1e-15)
    zero, _ = oracle_mod.short_conv(np.zeros((1, 3, 2)), np.ones((2, 4)), silu=True)
    assert np.array_equal(zero, np.zeros((1, 3, 2)))  # SiLU(0) = 0


def test_short_conv_continuation(oracle_mod):
    """A sequence cut in pieces, each started from the state the previous
    piece left, gives the uncut result, pieces shorter than W - 1 included."""
    rng = np.random.default_rng(72)
    cu, x, w, st = _conv_case(rng, [14], W=4)
    y, s = oracle_mod.short_conv(x, w, cu_seqlens=cu, state=st)
    parts, state = [], st
    for a, b in ((0, 5), (5, 6), (6, 8), (8, 8), (8, 14)):
        yp, state = oracle_mod.short_conv(x[a:b], w, cu_seqlens=np.array([0, b - a]), state=state)
        parts.append(yp)
    assert np.array_equal(np.concatenate(parts), y) and np.array_equal(state, s)


def test_short_conv_batched_equals_packed(oracle_mod):
    """The batched layout [B, T, ...] is the packed one with equal lengths."""
    rng = np.random.default_rng(73)
    x = rng.standard_normal((3, 7, 2, 3))
    w = rng.standard_normal((2, 3, 4))
    st = rng.standard_normal((3, 2, 3, 3))
    yb, sb = oracle_mod.short_conv(x, w, state=st)
    yp, sp = oracle_mod.short_conv(x.reshape(21, 2, 3), w, cu_seqlens=np.array([0, 7, 14, 21]), state=st)
    assert np.array_equal(yb.reshape(21, 2, 3), yp) and np.array_equal(sb, sp)


def test_conv_input_side_composition(oracle_mod):
    """The composed input side: with width-1 unit filters and the SiLU
    undone it is the L2 normalisation alone; each output row of q and k has
    unit norm; v is the SiLU of the convolution; a prefill's conv states
    carry a continuation exactly."""
    from scipy.special import expit
    rng = np.random.default_rng(74)
    T, hk, hv, dk, dv, W = 11, 2, 4, 8, 6, 4
    q = rng.standard_normal((1, T, hk, dk))
    k = rng.standard_normal((1, T, hk, dk))
    v = rng.standard_normal((1, T, hv, dv))
    wq, wk, wv = (rng.standard_normal((h, d, W)) for h, d in ((hk, dk), (hk, dk), (hv, dv)))
    qn, kn, vc, st = oracle_mod.conv_input_side(q, k, v, wq, wk, wv)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(kn, axis=-1), 1.0, rtol=0, atol=1e-12)
    plain_v, _ = oracle_mod.short_conv(v, wv, silu=False)
    assert np.allclose(vc, plain_v * expit(plain_v), rtol=1e-13, atol=1e-15)
    # width-1 unit filters: conv = identity, so q -> L2(SiLU(q)); compare against prepare on SiLU(q)
    one_q, one_k, one_v = np.ones((hk, dk, 1)), np.ones((hk, dk, 1)), np.ones((hv, dv, 1))
    q1, k1, v1, _ = oracle_mod.conv_input_side(q, k, v, one_q, one_k, one_v)
    sq, sk = q * expit(q), k * expit(k)
    pq, pk, _, _ = oracle_mod.prepare_inputs(sq, sk, np.zeros((1, T, 1)), np.zeros((1, T, 1)), qk_l2norm=True)
    assert np.allclose(q1, pq, rtol=1e-13, atol=1e-15) and np.allclose(k1, pk, rtol=1e-13, atol=1e-15)
    assert np.allclose(v1, v * expit(v), rtol=1e-13, atol=1e-15)
    # a prefill of the first 7 tokens, then the rest from its conv states
    a = oracle_mod.conv_input_side(q[:, :7], k[:, :7], v[:, :7], wq, wk, wv)
    b = oracle_mod.conv_input_side(q[:, 7:], k[:, 7:], v[:, 7:], wq, wk, wv, states=a[3])
    for i in range(3):
        assert np.array_equal(np.concatenate([a[i], b[i]], axis=1), (qn, kn, vc)[i])
    for n in ("q", "k", "v"):
        assert np.array_equal(b[3][n], st[n])
