"""Pins for the fp64 CPU oracle (CPU only).

Each test checks the oracle against something other than itself: hand-worked
cases, closed forms of special cases, invariants of the delta rule, and
agreement between two different algorithms (the token scan and the chunked
WY rewrite). The pinned facts and the mistakes they catch:

P1  hand-worked cases (tests/golden/hand_cases.json), dk != dv: plumbing,
    scale, decay axis, transposes, per-sequence initial states.
P2  one-hot keys with beta = 1: each write overwrites one key row, which then
    decays by its own channel's gate -> decay axis, inclusive cumulative sum.
P3  delta-rule invariant k_t^T S_t = (1 - beta_t) k_t^T D_t S_{t-1} + beta_t v_t^T
    for unit keys; with beta = 1 it is k_t^T S_t = v_t^T -> decay-then-erase
    order and the beta on the erase term.
P4  beta = 0: o_t = scale (q_t * exp G_t)^T S_0; the erase-free recurrence
    equals the gated-linear-attention sum exactly; small beta reaches that sum
    to first order -> gate semantics.
P5  g = 0, beta = 1, orthonormal (rotated) keys: DeltaNet replaces the value
    stored along each key direction -> dense erase term.
P6  linearity in (V, S_0) jointly and in scale; value-column independence.
P7  a packed batch equals its sequences run one by one (incl. empty and
    one-token sequences).
P8  resume: run(T1) then run(T2) from the final state equals run(T1 + T2).
P9  the naive chunked WY rewrite equals the scan (chunk sizes 1..64, ragged
    tails); the doubling inverse equals forward substitution.
P10 gate preprocessing (preprocess): unit norms per (token, head) over the
    channel axis and agreement with the input generator's own float32
    normalisation -> normalisation axis, missing square root; the exact
    identities log sigmoid(x) - log sigmoid(-x) = x and
    sigmoid(x) + sigmoid(-x) = 1, log sigmoid(0) = -log 2 -> sign errors,
    wrong branch of the stable form; the lower bound clamps exactly where
    log sigmoid falls below it; agreement with the generator's gates and
    betas computed from the same draws.
P12 the time split's combination: the second part of a sequence run from a
    start state S_a equals the same part run from zero plus S_a applied to the
    part's transition map, o_t = o_loc(t) + S_a^T o_M(t) and S_T = M S_a + B,
    where o_M and M come from the part run with v = 0 from the identity ->
    which side S_a multiplies, the transpose in o, the scale inside o_M.
P13 the chunked (WY-form) backward equals the token-level reverse recurrence at
    chunk sizes 1..32 -> every term of the chunked derivative (the adjoint
    state step, the inverse's derivative, the masks, the decay chain rule
    and the in-chunk reverse cumulative sum).
P11 backward: the reverse-mode gradients of q, k, v, g, beta and the initial
    state equal central finite differences of the (pinned) forward scan, per
    coordinate and along random directions -> every term of the hand-derived
    reverse recurrence (a dropped term, a wrong sign or transpose shows as a
    gradient mismatch).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _frac_array(x):
    return np.array([[float(Fraction(s)) for s in row] for row in x], dtype=np.float64)


def _rand_f64(seqlens, H, dk, dv, seed, *, gmin=-5.0, unit_keys=True, init=False):
    rng = np.random.default_rng(seed)
    T = int(sum(seqlens))
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    g = rng.uniform(gmin, 0.0, size=(T, H, dk))
    beta = rng.uniform(0.05, 1.0, size=(T, H))
    cu = np.zeros(len(seqlens) + 1, np.int32)
    cu[1:] = np.cumsum(seqlens)
    S0 = rng.standard_normal((len(seqlens), H, dk, dv)) * 0.3 if init else None
    return q, k, v, g, beta, cu, S0


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


# ----------------------------------------------------------------------------- P1
def test_p1_hand_cases(oracle_mod):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 3
    for c in cases:
        dk, dv = c["dk"], c["dv"]
        T = len(c["q"])
        seqlens = c.get("seqlens", [T])
        cu = np.zeros(len(seqlens) + 1, np.int32)
        cu[1:] = np.cumsum(seqlens)
        q = _frac_array(c["q"]).reshape(T, 1, dk)
        k = _frac_array(c["k"]).reshape(T, 1, dk)
        v = _frac_array(c["v"]).reshape(T, 1, dv)
        g = np.log(_frac_array(c["decay"])).reshape(T, 1, dk)
        beta = np.array([float(Fraction(s)) for s in c["beta"]]).reshape(T, 1)
        S0 = None
        if c["initial_state"] is not None:
            S0 = np.array(c["initial_state"], dtype=object)
            S0 = np.vectorize(lambda s: float(Fraction(s)))(S0).astype(np.float64)
            S0 = S0.reshape(len(seqlens), 1, dk, dv)
        out, fin = oracle_mod.scan(q, k, v, g, beta, cu, float(Fraction(c["scale"])), S0)
        exp_out = _frac_array(c["expected_out"]).reshape(T, 1, dv)
        exp_fin = np.vectorize(lambda s: float(Fraction(s)))(np.array(c["expected_final"], dtype=object))
        exp_fin = exp_fin.astype(np.float64).reshape(len(seqlens), 1, dk, dv)
        np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(fin, exp_fin, rtol=0, atol=1e-14, err_msg=c["name"])


# ----------------------------------------------------------------------------- P2
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_p2_one_hot_keys_closed_form(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    T, dk, dv = 37, 8, 5
    idx = rng.integers(0, dk - 2, size=T)  # keys dk-2, dk-1 never written
    k = np.zeros((T, 1, dk))
    k[np.arange(T), 0, idx] = 1.0
    q = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    g = rng.uniform(-1.0, 0.0, size=(T, 1, dk))
    beta = np.ones((T, 1))
    S0 = rng.standard_normal((1, 1, dk, dv))
    cu = np.array([0, T], np.int32)
    scale = 0.7
    out, fin = oracle_mod.scan(q, k, v, g, beta, cu, scale, S0)
    G = np.cumsum(g[:, 0, :], axis=0)  # inclusive cumulative log-decay
    for t in range(T):
        S = np.empty((dk, dv))
        for j in range(dk):
            writes = [s for s in range(t + 1) if idx[s] == j]
            if writes:
                tau = writes[-1]
                S[j] = np.exp(G[t, j] - G[tau, j]) * v[tau, 0]
            else:
                S[j] = np.exp(G[t, j]) * S0[0, 0, j]
        np.testing.assert_allclose(out[t, 0], scale * S.T @ q[t, 0], rtol=1e-12, atol=1e-13)
        if t == T - 1:
            np.testing.assert_allclose(fin[0, 0], S, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- P3
def test_p3_delta_rule_invariant(oracle_mod):
    q, k, v, g, beta, cu, S0 = _rand_f64([24], 1, 16, 6, seed=3, init=True)
    # prefix runs give S_t for every t
    states = []
    for t in range(1, 25):
        _, fin = oracle_mod.scan(q[:t], k[:t], v[:t], g[:t], beta[:t], np.array([0, t], np.int32), 1.0, S0)
        states.append(fin[0, 0])
    prev = S0[0, 0]
    for t in range(24):
        kt, bt = k[t, 0], beta[t, 0]
        DS = np.exp(g[t, 0])[:, None] * prev
        lhs = kt @ states[t]
        rhs = (1.0 - bt) * (kt @ DS) + bt * v[t, 0]
        np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-13)
        prev = states[t]
    # beta = 1: the state answers the last key with the last value exactly
    beta1 = np.ones_like(beta)
    for t in (1, 7, 24):
        _, fin = oracle_mod.scan(q[:t], k[:t], v[:t], g[:t], beta1[:t], np.array([0, t], np.int32), 1.0, S0)
        np.testing.assert_allclose(k[t - 1, 0] @ fin[0, 0], v[t - 1, 0], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- P4
def _gla_sum(q, k, v, g, beta, S0, scale):
    T, H, dk = q.shape
    out = np.zeros((T, H, v.shape[2]))
    for h in range(H):
        G = np.cumsum(g[:, h, :], axis=0)
        for t in range(T):
            acc = (q[t, h] * np.exp(G[t])) @ S0[h] if S0 is not None else 0.0
            for s in range(t + 1):
                acc = acc + ((q[t, h] * np.exp(G[t] - G[s])) @ k[s, h]) * beta[s, h] * v[s, h]
            out[t, h] = scale * acc
    return out


def test_p4_beta_zero_closed_form(oracle_mod):
    q, k, v, g, beta, cu, S0 = _rand_f64([20], 2, 8, 4, seed=4, init=True)
    out, fin = oracle_mod.scan(q, k, v, g, np.zeros_like(beta), cu, 0.5, S0)
    G = np.cumsum(g, axis=0)
    for h in range(2):
        for t in range(20):
            np.testing.assert_allclose(out[t, h], 0.5 * (q[t, h] * np.exp(G[t, h])) @ S0[0, h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(fin[0, h], np.exp(G[-1, h])[:, None] * S0[0, h], rtol=1e-12, atol=1e-14)


def test_p4_erase_free_equals_gla_sum(oracle_mod):
    q, k, v, g, beta, cu, S0 = _rand_f64([18], 2, 8, 5, seed=5, init=True)
    out, _ = oracle_mod.scan(q, k, v, g, beta, cu, 0.3, S0, erase=False)
    ref = _gla_sum(q, k, v, g, beta, S0[0], 0.3)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_p4_small_beta_reaches_gla_sum(oracle_mod):
    q, k, v, g, beta, cu, _ = _rand_f64([16], 1, 8, 4, seed=6)
    eps = 1e-6
    out, _ = oracle_mod.scan(q, k, v, g, np.full_like(beta, eps), cu, 1.0, None)
    ref = _gla_sum(q, k, v, g, np.ones_like(beta), None, 1.0)
    # the erase term is O(eps^2): o / eps = GLA sum + O(eps)
    assert _rel(out / eps, ref) < 1e-4


# ----------------------------------------------------------------------------- P5
def test_p5_deltanet_orthonormal_keys(oracle_mod):
    rng = np.random.default_rng(7)
    dk, dv, T = 6, 3, 25
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))  # orthonormal basis (columns)
    idx = rng.integers(0, dk - 1, size=T)                # direction dk-1 never written
    k = Qm[:, idx].T.reshape(T, 1, dk)
    q = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    S0 = rng.standard_normal((1, 1, dk, dv))
    out, fin = oracle_mod.scan(q, k, v, np.zeros((T, 1, dk)), np.ones((T, 1)), np.array([0, T], np.int32), 1.0, S0)
    S = np.zeros((dk, dv))
    for j in range(dk):
        b = Qm[:, j]
        writes = [s for s in range(T) if idx[s] == j]
        S += np.outer(b, v[writes[-1], 0] if writes else b @ S0[0, 0])
    np.testing.assert_allclose(fin[0, 0], S, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out[-1, 0], S.T @ q[-1, 0], rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------- P6
def test_p6_linearity_and_column_independence(oracle_mod):
    q, k, v, g, beta, cu, S0 = _rand_f64([11, 0, 17], 2, 8, 6, seed=8, init=True)
    rng = np.random.default_rng(9)
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    a, b = 0.75, -1.5
    o1, f1 = oracle_mod.scan(q, k, v, g, beta, cu, 0.4, S0)
    o2, f2 = oracle_mod.scan(q, k, v2, g, beta, cu, 0.4, S02)
    o3, f3 = oracle_mod.scan(q, k, a * v + b * v2, g, beta, cu, 0.4, a * S0 + b * S02)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(f3, a * f1 + b * f2, rtol=1e-11, atol=1e-12)
    o4, _ = oracle_mod.scan(q, k, v, g, beta, cu, 1.2, S0)
    np.testing.assert_allclose(o4, o1 * 3.0, rtol=1e-12, atol=1e-14)
    # value columns evolve independently: a run on a column slice (its own v and
    # S0 columns) reproduces those columns of the full run bit for bit
    cs = slice(2, 5)
    o5, f5 = oracle_mod.scan(q, k, np.ascontiguousarray(v[:, :, cs]), g, beta, cu, 0.4,
                             np.ascontiguousarray(S0[..., cs]))
    assert np.array_equal(o5, o1[:, :, cs]) and np.array_equal(f5, f1[..., cs])
    for blk in (1, 4, 6):
        o6, f6 = oracle_mod.scan(q, k, v, g, beta, cu, 0.4, S0, col_block=blk)
        assert np.array_equal(o6, o1) and np.array_equal(f6, f1)


# ----------------------------------------------------------------------------- P7
def test_p7_varlen_equals_separate_sequences(oracle_mod):
    lens = [5, 0, 1, 13, 0, 9]
    q, k, v, g, beta, cu, S0 = _rand_f64(lens, 2, 8, 4, seed=10, init=True)
    out, fin = oracle_mod.scan(q, k, v, g, beta, cu, 0.6, S0)
    for i, L in enumerate(lens):
        t0, t1 = cu[i], cu[i + 1]
        o_i, f_i = oracle_mod.scan(q[t0:t1], k[t0:t1], v[t0:t1], g[t0:t1], beta[t0:t1],
                                   np.array([0, L], np.int32), 0.6, S0[i:i + 1])
        assert np.array_equal(out[t0:t1], o_i)
        assert np.array_equal(fin[i], f_i[0])
        if L == 0:
            assert np.array_equal(fin[i], S0[i])


# ----------------------------------------------------------------------------- P8
def test_p8_resume_from_final_state(oracle_mod):
    q, k, v, g, beta, cu, S0 = _rand_f64([30], 2, 8, 4, seed=11, init=True)
    out, fin = oracle_mod.scan(q, k, v, g, beta, cu, 0.5, S0)
    for T1 in (1, 13, 29):
        oa, fa = oracle_mod.scan(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], np.array([0, T1], np.int32), 0.5, S0)
        ob, fb = oracle_mod.scan(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], np.array([0, 30 - T1], np.int32), 0.5, fa)
        assert np.array_equal(np.concatenate([oa, ob]), out)
        assert np.array_equal(fb, fin)


# ----------------------------------------------------------------------------- P12
@pytest.mark.parametrize("T1", [1, 9, 20])
def test_p12_time_split_combination(oracle_mod, T1):
    d, T, H, scale = 8, 29, 2, 0.7
    q, k, v, g, beta, cu, S0 = _rand_f64([T], H, d, d, seed=40 + T1, init=True)
    out, fin = oracle_mod.scan(q, k, v, g, beta, cu, scale, S0)
    part = lambda x: np.ascontiguousarray(x[T1:])
    cu2 = np.array([0, T - T1], np.int32)
    # first part from the initial state
    oa, Sa = oracle_mod.scan(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], np.array([0, T1], np.int32), scale, S0)
    # second part from zero, and with v = 0 from the identity (its transition map)
    oloc, B = oracle_mod.scan(part(q), part(k), part(v), part(g), part(beta), cu2, scale, None)
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    oM, M = oracle_mod.scan(part(q), part(k), np.zeros_like(part(v)), part(g), part(beta), cu2, scale, eye)
    # combine: per head h, o_t = o_loc(t) + S_a[h]^T o_M(t); S_T = M[h] S_a[h] + B[h]
    o2 = oloc + np.einsum("hkv,thk->thv", Sa[0], oM)
    f2 = np.einsum("hij,hjv->hiv", M[0], Sa[0]) + B[0]
    np.testing.assert_allclose(np.concatenate([oa, o2]), out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f2, fin[0], rtol=1e-10, atol=1e-12)
    # the transposed combination is wrong (the pin distinguishes the two)
    wrong = oloc + np.einsum("hvk,thk->thv", Sa[0], oM)
    assert np.max(np.abs(wrong - out[T1:])) > 1e-3


# ----------------------------------------------------------------------------- P13
@pytest.mark.parametrize("chunk", [1, 5, 16, 32])
@pytest.mark.parametrize("with_state", [False, True])
def test_p13_chunked_backward_equals_token_backward(oracle_mod, chunk, with_state):
    lens = [37, 0, 16, 5]
    q, k, v, g, beta, cu, S0 = _rand_f64(lens, 2, 6, 5, seed=50 + chunk, init=with_state)
    rng = np.random.default_rng(51)
    dout = rng.standard_normal(v.shape)
    dfin = rng.standard_normal((len(lens), 2, 6, 5)) if with_state else None
    ref = oracle_mod.backward(q, k, v, g, beta, cu, 0.5, dout, S0, dfin)
    got = oracle_mod.chunked_backward(q, k, v, g, beta, cu, 0.5, dout, S0, dfin, chunk=chunk)
    for name in ("dq", "dk", "dv", "dg", "dbeta") + (("dinit",) if with_state else ()):
        assert _rel(got[name], ref[name]) < 1e-10, name


# ----------------------------------------------------------------------------- P9
@pytest.mark.parametrize("chunk", [1, 4, 7, 16, 32, 64])
def test_p9_chunked_equals_scan(oracle_mod, chunk):
    lens = [1, 31, 64, 100, 0, 65]
    q, k, v, g, beta, cu, S0 = _rand_f64(lens, 2, 16, 8, seed=12 + chunk, init=True)
    o_s, f_s = oracle_mod.scan(q, k, v, g, beta, cu, 0.25, S0)
    o_c, f_c = oracle_mod.chunked(q, k, v, g, beta, cu, 0.25, S0, chunk=chunk)
    assert _rel(o_c, o_s) < 1e-12
    assert _rel(f_c, f_s) < 1e-12


def test_p9_chunked_equals_scan_library_inputs(oracle_mod):
    import kda_inputs

    inp = kda_inputs.make_inputs([70, 3, 129], 2, seed=5, random_initial_state=True)
    o_s, f_s = oracle_mod.scan_inputs(inp)
    o_c, f_c = oracle_mod.chunked(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.scale,
                                  inp.initial_state, chunk=64)
    assert _rel(o_c, o_s) < 1e-12 and _rel(f_c, f_s) < 1e-12


@pytest.mark.parametrize("n", [2, 5, 16, 32, 64])
def test_p9_doubling_inverse(oracle_mod, n):
    rng = np.random.default_rng(n)
    L = np.tril(rng.uniform(-0.5, 0.5, size=(n, n)), -1)
    X = oracle_mod.unit_lower_inverse(L, "substitution")
    np.testing.assert_allclose((np.eye(n) + L) @ X, np.eye(n), atol=1e-12)
    Xd = oracle_mod.unit_lower_inverse(L, "doubling")
    np.testing.assert_allclose(Xd, X, rtol=1e-12, atol=1e-12)
    # nilpotency that the doubling relies on: L^n = 0 for strictly lower n x n
    assert np.max(np.abs(np.linalg.matrix_power(L, n))) == 0.0


def test_oracle_rejects_bad_cu_seqlens(oracle_mod):
    q, k, v, g, beta, cu, _ = _rand_f64([4, 4], 1, 4, 4, seed=1)
    with pytest.raises(ValueError):
        oracle_mod.scan(q, k, v, g, beta, np.array([0, 5, 4], np.int32), 1.0)
    with pytest.raises(ValueError):
        oracle_mod.scan(q, k, v, g, beta, np.array([0, 4, 9], np.int32), 1.0)


def test_inputs_generator_is_deterministic_and_shaped():
    import kda_inputs

    a = kda_inputs.make_inputs([7, 0, 5], 3, seed=42, random_initial_state=True)
    b = kda_inputs.make_inputs([7, 0, 5], 3, seed=42, random_initial_state=True, row_block=2)
    for name in ("q", "k", "v", "g", "beta", "cu_seqlens", "initial_state"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    assert a.q.shape == (12, 3, 128) and a.q.dtype == np.uint16
    assert a.g.dtype == np.float32 and a.g.min() >= -5.0 and a.g.max() <= 0.0
    assert a.beta.min() > 0 and a.beta.max() < 1
    kf = kda_inputs.bf16_bits_to_f32(a.k)
    assert np.allclose(np.linalg.norm(kf, axis=-1), 1.0, atol=1e-2)
    assert list(a.cu_seqlens) == [0, 7, 7, 12]
    # round-to-nearest-even on exactly representable halfway cases
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32)
    assert list(kda_inputs.bf16_bits_to_f32(kda_inputs.f32_to_bf16_bits(x))) == [1.0, 1.0 + 2 ** -6]


# ----------------------------------------------------------------------------- P10
def _raw_batch(seed=40):
    import kda_inputs

    return kda_inputs.make_inputs([33, 0, 70], 3, seed=seed, raw=True, random_initial_state=True)


def test_p10_normalisation_unit_norm_and_generator_agreement(oracle_mod):
    import kda_inputs

    inp = _raw_batch()
    qh, kh, _, _ = oracle_mod.preprocess(inp.q_raw, inp.k_raw, inp.g_logit, inp.beta_logit)
    for x in (qh, kh):
        assert np.allclose(np.linalg.norm(x, axis=-1), 1.0, rtol=0, atol=1e-14)
    # the generator normalised the unrounded float32 draws, then rounded to
    # bf16; the oracle normalises the bf16-rounded draws in fp64. Per element
    # the two differ by at most three bf16 roundings (the draw's, its effect on
    # the norm, the generator's output), each at most 2^-8 relative
    for x, ref in ((qh, inp.q), (kh, inp.k)):
        r = kda_inputs.bf16_bits_to_f32(ref).astype(np.float64)
        assert np.all(np.abs(x - r) <= 3 * 2.0 ** -8 * np.abs(r) + 1e-7)
    # a zero row stays zero (the norm is floored at eps), a scaled row gives the same direction
    qz = inp.q_raw.copy()
    qz[0, 0, :] = 0
    qz[1, 1, :] = kda_inputs.f32_to_bf16_bits(4.0 * kda_inputs.bf16_bits_to_f32(inp.q_raw[1, 1]))
    qh2, _, _, _ = oracle_mod.preprocess(qz, inp.k_raw, inp.g_logit, inp.beta_logit)
    assert np.all(qh2[0, 0] == 0.0)
    assert np.allclose(qh2[1, 1], qh[1, 1], rtol=0, atol=1e-15)


def test_p10_gate_identities_and_lower_bound(oracle_mod):
    x = np.array([[[-100.0, -30.0, -5.5, -1.0, -1e-3, 0.0, 1e-3, 0.7, 3.0, 25.0, 90.0, 200.0]]], np.float32)
    T, H, dk = x.shape
    q = np.full((T, H, dk), 0x3F80, np.uint16)  # bf16 1.0
    b = np.array([[-3.0]], np.float32)
    _, _, g_pos, beta_pos = oracle_mod.preprocess(q, q, x, b, lower_bound=-1e300)
    _, _, g_neg, beta_neg = oracle_mod.preprocess(q, q, -x, -b, lower_bound=-1e300)
    xd = x.astype(np.float64)
    assert np.allclose(g_pos - g_neg, xd, rtol=1e-15, atol=1e-13)          # ls(x) - ls(-x) = x
    assert np.allclose(np.exp(g_pos) + np.exp(g_neg), 1.0, rtol=0, atol=1e-15)
    assert g_pos[0, 0, 5] == -np.log(2.0)
    assert np.all(g_pos <= 0.0)
    assert abs(beta_pos[0, 0] + beta_neg[0, 0] - 1.0) < 1e-15 and beta_pos[0, 0] < 0.5
    # the lower bound replaces exactly the values below it
    _, _, g5, _ = oracle_mod.preprocess(q, q, x, b, lower_bound=-5.0)
    below = g_pos < -5.0
    assert np.all(g5[below] == -5.0) and np.all(g5[~below] == g_pos[~below])
    assert below.sum() == 3  # x = -100, -30, -5.5


def test_p10_gates_and_betas_agree_with_generator(oracle_mod):
    inp = _raw_batch(41)
    _, _, g, beta = oracle_mod.preprocess(inp.q_raw, inp.k_raw, inp.g_logit, inp.beta_logit)
    # the generator computed from the unrounded float64 logits and rounded
    # its results to float32; the logits here are their float32 roundings
    assert np.max(np.abs(g - inp.g.astype(np.float64))) <= 1e-5
    assert np.max(np.abs(beta - inp.beta.astype(np.float64))) <= 1e-6


def test_p10_preprocessed_scan_matches_generator_scan(oracle_mod):
    """The scan on preprocessed raw draws and the scan on the generator's
    inputs differ only by the generator's bf16 rounding of q and k."""
    inp = _raw_batch(42)
    o1, f1 = oracle_mod.scan_raw_inputs(inp)
    o2, f2 = oracle_mod.scan_inputs(inp)
    assert np.linalg.norm(o1 - o2) / np.linalg.norm(o2) < 1e-2
    assert np.linalg.norm(f1 - f2) / np.linalg.norm(f2) < 1e-2


# ----------------------------------------------------------------------------- P11
def _loss(oracle_mod, args, dout, dfin):
    q, k, v, g, beta, cu, S0, scale = args
    o, f = oracle_mod.scan(q, k, v, g, beta, cu, scale, S0)
    return float(np.sum(o * dout) + np.sum(f * dfin))


@pytest.mark.parametrize("seed", [0, 1])
def test_p11_backward_equals_finite_differences(oracle_mod, seed):
    lens, H, dk, dv = [5, 0, 9, 1], 2, 6, 5
    q, k, v, g, beta, cu, S0 = _rand_f64(lens, H, dk, dv, 70 + seed, gmin=-2.0, init=True)
    scale = 0.7
    rng = np.random.default_rng(80 + seed)
    dout = rng.standard_normal(v.shape)
    dfin = rng.standard_normal(S0.shape)
    gr = oracle_mod.backward(q, k, v, g, beta, cu, scale, dout, S0, dfin)
    base = [q, k, v, g, beta, cu, S0, scale]
    names = {"dq": 0, "dk": 1, "dv": 2, "dg": 3, "dbeta": 4, "dinit": 6}
    h = 1e-6
    for name, idx in names.items():
        x = base[idx]
        # a handful of single coordinates
        flat = rng.choice(x.size, size=min(6, x.size), replace=False)
        for f in flat:
            plus = [a.copy() if isinstance(a, np.ndarray) else a for a in base]
            minus = [a.copy() if isinstance(a, np.ndarray) else a for a in base]
            plus[idx].flat[f] += h
            minus[idx].flat[f] -= h
            fd = (_loss(oracle_mod, plus, dout, dfin) - _loss(oracle_mod, minus, dout, dfin)) / (2 * h)
            an = gr[name].flat[f]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, f, fd, an)
        # one random direction over all coordinates
        d = rng.standard_normal(x.shape)
        plus = [a.copy() if isinstance(a, np.ndarray) else a for a in base]
        minus = [a.copy() if isinstance(a, np.ndarray) else a for a in base]
        plus[idx] = plus[idx] + h * d
        minus[idx] = minus[idx] - h * d
        fd = (_loss(oracle_mod, plus, dout, dfin) - _loss(oracle_mod, minus, dout, dfin)) / (2 * h)
        an = float(np.sum(gr[name] * d))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, "direction", fd, an)


def test_p11_backward_long_sequence_crosses_checkpoints(oracle_mod):
    """The oracle recomputes states from checkpoints every 64 tokens; a
    sequence over several checkpoints gives the finite-difference gradients."""
    lens, H, dk, dv = [150], 1, 4, 3
    q, k, v, g, beta, cu, S0 = _rand_f64(lens, H, dk, dv, 90, gmin=-0.3, init=True)
    rng = np.random.default_rng(91)
    dout = rng.standard_normal(v.shape)
    dfin = rng.standard_normal(S0.shape)
    gr = oracle_mod.backward(q, k, v, g, beta, cu, 0.5, dout, S0, dfin)
    base = [q, k, v, g, beta, cu, S0, 0.5]
    h = 1e-6
    for name, idx in {"dk": 1, "dg": 3, "dinit": 6}.items():
        d = rng.standard_normal(base[idx].shape)
        plus = list(base)
        minus = list(base)
        plus[idx] = base[idx] + h * d
        minus[idx] = base[idx] - h * d
        fd = (_loss(oracle_mod, plus, dout, dfin) - _loss(oracle_mod, minus, dout, dfin)) / (2 * h)
        an = float(np.sum(gr[name] * d))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)
