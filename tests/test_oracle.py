"""Pins for the CPU oracle: each check ties it to something other than itself.

The token recurrence is pinned by the brute-force transition-matrix form, by
closed forms (beta = 0, one token, scalar state, unit keys, orthonormal keys)
and by structural facts (GQA grouping, varlen packing, split/resume).  The
chunked form is pinned to the token form (relative Frobenius <= 1e-10) and to
chunk-size independence.  Verify/fold is pinned to sequential steps, BA gates
to numpy/scipy library routines and to the slot table the BA page defines.
"""
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_frob(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def rand_problem(rng, seqlens, H_k, H_v, d_k, d_v, h0=True, g_scale=1.0):
    T = sum(seqlens)
    q = rng.standard_normal((T, H_k, d_k))
    k = rng.standard_normal((T, H_k, d_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, d_v))
    g = -np.abs(rng.standard_normal((T, H_v))) * 0.3 * g_scale
    beta = rng.uniform(0.05, 0.95, (T, H_v))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    hs = rng.standard_normal((len(seqlens), H_v, d_k, d_v)) * 0.3 if h0 else None
    return q, k, v, g, beta, cu, hs


# --------------------------------------------------------------------------
# Token recurrence vs brute force (explicit transition matrices, long double)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", range(6))
def test_token_matches_brute_force(case):
    rng = np.random.default_rng(100 + case)
    d_k, d_v = int(rng.integers(2, 6)), int(rng.integers(1, 5))
    H_k = int(rng.integers(1, 3))
    H_v = H_k * int(rng.integers(1, 3))
    seqlens = [int(x) for x in rng.integers(1, 9, size=int(rng.integers(1, 3)))]
    q, k, v, g, beta, cu, h0 = rand_problem(rng, seqlens, H_k, H_v, d_k, d_v)
    # positive gates too: the definition does not need g <= 0
    g = g + rng.uniform(-0.2, 0.2, g.shape)
    o1, h1 = oracle.gdn_token(q, k, v, g, beta, cu, h0, scale=0.7)
    o2, h2 = oracle.gdn_brute(q, k, v, g, beta, cu, h0, scale=0.7)
    assert rel_frob(o1, o2) <= 1e-12
    assert rel_frob(h1, h2) <= 1e-12


def test_brute_force_against_numpy_products():
    """The brute-force form itself, re-derived with numpy matrix products."""
    rng = np.random.default_rng(7)
    T, d_k, d_v = 5, 3, 2
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [T], 1, 1, d_k, d_v)
    o, hT = oracle.gdn_brute(q, k, v, g, beta, cu, h0)
    S = h0[0, 0].T.copy()  # S_0 = H0^T, [d_v, d_k]
    for t in range(T):
        kt = k[t, 0]
        M = np.exp(g[t, 0]) * (np.eye(d_k) - beta[t, 0] * np.outer(kt, kt))
        S = S @ M + beta[t, 0] * np.outer(v[t, 0], kt)
        np.testing.assert_allclose(o[t, 0], S @ q[t, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], S.T, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def test_beta_zero_only_decays():
    """beta = 0: S_T = exp(sum g) S_0 and o_t = exp(G_t) S_0 q_t."""
    rng = np.random.default_rng(1)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [37], 2, 4, 8, 6)
    beta[:] = 0.0
    o, hT = oracle.gdn_token(q, k, v, g, beta, cu, h0)
    G = np.cumsum(g, axis=0)  # [T, H_v]
    for h in range(4):
        S0 = h0[0, h].T
        np.testing.assert_allclose(hT[0, h], np.exp(G[-1, h]) * h0[0, h], rtol=1e-13)
        for t in range(37):
            np.testing.assert_allclose(o[t, h], np.exp(G[t, h]) * S0 @ q[t, h // 2],
                                       rtol=1e-12, atol=1e-15)


def test_unit_key_writes_value_column():
    """g = 0, beta = 1, k = e_j: S e_j becomes v, every other column is kept."""
    rng = np.random.default_rng(2)
    d_k, d_v = 5, 3
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [1], 1, 1, d_k, d_v)
    j = 3
    k[:] = 0.0
    k[0, 0, j] = 1.0
    g[:] = 0.0
    beta[:] = 1.0
    _, hT = oracle.gdn_token(q, k, v, g, beta, cu, h0)
    S0, S1 = h0[0, 0].T, hT[0, 0].T
    np.testing.assert_allclose(S1[:, j], v[0, 0], rtol=1e-14)
    others = [c for c in range(d_k) if c != j]
    np.testing.assert_array_equal(S1[:, others], S0[:, others])


def test_single_token_closed_form():
    rng = np.random.default_rng(3)
    d_k, d_v = 6, 4
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [1], 1, 1, d_k, d_v)
    o, hT = oracle.gdn_token(q, k, v, g, beta, cu, h0, scale=1.3)
    S0 = h0[0, 0].T
    kk, qq, vv = k[0, 0], q[0, 0], v[0, 0]
    gam, b = np.exp(g[0, 0]), beta[0, 0]
    S1 = gam * S0 + b * np.outer(vv - gam * S0 @ kk, kk)
    np.testing.assert_allclose(hT[0, 0], S1.T, rtol=1e-13)
    np.testing.assert_allclose(o[0, 0], 1.3 * S1 @ qq, rtol=1e-13)


def test_scalar_state_recurrence():
    """d_k = d_v = 1: s_t = e^{g} s (1 - beta k^2) + beta v k, o_t = s_t q_t."""
    rng = np.random.default_rng(4)
    T = 50
    q = rng.standard_normal((T, 1, 1))
    k = rng.standard_normal((T, 1, 1))
    v = rng.standard_normal((T, 1, 1))
    g = -rng.uniform(0, 0.5, (T, 1))
    beta = rng.uniform(0, 1, (T, 1))
    h0 = np.array([[[[0.4]]]])
    o, hT = oracle.gdn_token(q, k, v, g, beta, [0, T], h0)
    s = 0.4
    for t in range(T):
        kt = k[t, 0, 0]
        s = np.exp(g[t, 0]) * s * (1 - beta[t, 0] * kt * kt) + beta[t, 0] * v[t, 0, 0] * kt
        assert o[t, 0, 0] == pytest.approx(s * q[t, 0, 0], rel=1e-12, abs=1e-15)
    assert hT[0, 0, 0, 0] == pytest.approx(s, rel=1e-12)


def test_orthonormal_keys_store_values():
    """beta = 1, g = 0, keys e_0..e_{T-1}: S_T = S_0 (I - sum e e^T) + sum v e^T."""
    rng = np.random.default_rng(5)
    d_k, d_v, T = 7, 3, 4
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [T], 1, 1, d_k, d_v)
    k[:] = 0.0
    for t in range(T):
        k[t, 0, t] = 1.0
    g[:] = 0.0
    beta[:] = 1.0
    _, hT = oracle.gdn_token(q, k, v, g, beta, cu, h0)
    P = np.zeros((d_k, d_k))
    E = np.zeros((d_v, d_k))
    for t in range(T):
        P[t, t] = 1.0
        E[:, t] = v[t, 0]
    want = h0[0, 0].T @ (np.eye(d_k) - P) + E
    np.testing.assert_allclose(hT[0, 0], want.T, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# Structure: GQA grouping, varlen packing, split/resume
# --------------------------------------------------------------------------

def test_gqa_grouping_is_contiguous():
    """v-head h reads k-head h // (H_v/H_k): same as repeating q/k per v-head."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [29], 2, 6, 5, 4)
    o1, h1 = oracle.gdn_token(q, k, v, g, beta, cu, h0)
    qr, kr = np.repeat(q, 3, axis=1), np.repeat(k, 3, axis=1)
    o2, h2 = oracle.gdn_token(qr, kr, v, g, beta, cu, h0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(h1, h2)


def test_varlen_packing_equals_separate_calls():
    rng = np.random.default_rng(8)
    lens = [17, 64, 1, 90]
    q, k, v, g, beta, cu, h0 = rand_problem(rng, lens, 2, 4, 8, 8)
    o, hT = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=16)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        on, hn = oracle.gdn_token(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], [0, b - a],
                                  h0[n:n + 1])
        assert rel_frob(o[a:b], on) <= 1e-10
        assert rel_frob(hT[n:n + 1], hn) <= 1e-10


def test_split_resume_equals_one_call():
    rng = np.random.default_rng(9)
    T, T1 = 150, 70
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [T], 1, 2, 8, 8)
    o, hT = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=64)
    o1, h1 = oracle.gdn_chunked(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], [0, T1], h0, chunk=64)
    o2, h2 = oracle.gdn_chunked(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], [0, T - T1], h1,
                                chunk=64)
    assert rel_frob(np.concatenate([o1, o2]), o) <= 1e-10
    assert rel_frob(h2, hT) <= 1e-10


def test_zero_initial_state_is_null_h0():
    rng = np.random.default_rng(10)
    q, k, v, g, beta, cu, _ = rand_problem(rng, [40], 1, 1, 4, 4, h0=False)
    o1, h1 = oracle.gdn_token(q, k, v, g, beta, cu, None)
    o2, h2 = oracle.gdn_token(q, k, v, g, beta, cu, np.zeros((1, 1, 4, 4)))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(h1, h2)


# --------------------------------------------------------------------------
# Chunked form vs token form
# --------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [1, 3, 16, 64])
def test_chunked_matches_token(chunk):
    rng = np.random.default_rng(11)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [200, 77], 2, 4, 16, 12)
    o1, h1 = oracle.gdn_token(q, k, v, g, beta, cu, h0, scale=0.5)
    o2, h2 = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, scale=0.5, chunk=chunk)
    assert rel_frob(o2, o1) <= 1e-10
    assert rel_frob(h2, h1) <= 1e-10


def test_chunked_matches_brute_force_short():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [8, 5], 1, 2, 4, 3)
    o1, h1 = oracle.gdn_brute(q, k, v, g, beta, cu, h0)
    o2, h2 = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=3)
    assert rel_frob(o2, o1) <= 1e-12
    assert rel_frob(h2, h1) <= 1e-12


def test_chunked_strong_decay_stays_finite():
    """Very negative gates (G down to about -700 in a chunk) keep every
    exponent of the chunked form <= 0: no overflow, same answer."""
    rng = np.random.default_rng(13)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [130], 1, 1, 8, 8)
    g[:] = -rng.uniform(5.0, 15.0, g.shape)
    o1, h1 = oracle.gdn_token(q, k, v, g, beta, cu, h0)
    o2, h2 = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=64)
    assert np.isfinite(o2).all() and np.isfinite(h2).all()
    assert rel_frob(o2, o1) <= 1e-10
    assert np.allclose(h2, h1, rtol=1e-10, atol=1e-300)


def test_chunk_size_independence():
    rng = np.random.default_rng(14)
    q, k, v, g, beta, cu, h0 = rand_problem(rng, [333], 1, 3, 12, 10)
    o1, h1 = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=64)
    o2, h2 = oracle.gdn_chunked(q, k, v, g, beta, cu, h0, chunk=7)
    assert rel_frob(o2, o1) <= 1e-10
    assert rel_frob(h2, h1) <= 1e-10


# --------------------------------------------------------------------------
# Verify / fold
# --------------------------------------------------------------------------

def _verify_problem(seed, batch=5, K=4, H_k=2, H_v=4, d_k=8, d_v=6):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, _, _ = rand_problem(rng, [batch * K], H_k, H_v, d_k, d_v, h0=False)
    hs = rng.standard_normal((batch, H_v, d_k, d_v)) * 0.2
    return q, k, v, g, beta, hs


def test_verify_outputs_are_sequential_steps():
    q, k, v, g, beta, hs = _verify_problem(20)
    na = np.zeros(5, dtype=np.int32)
    o, hf = oracle.gdn_verify_fold(hs, q, k, v, g, beta, na)
    for b in range(5):
        sl = slice(4 * b, 4 * b + 4)
        ob, _ = oracle.gdn_brute(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, 4], hs[b:b + 1])
        assert rel_frob(o[sl], ob) <= 1e-12
    np.testing.assert_array_equal(hf, hs)  # na = 0 everywhere: bit-identical


@pytest.mark.parametrize("na_all", [1, 2, 3, 4])
def test_fold_equals_na_sequential_steps(na_all):
    q, k, v, g, beta, hs = _verify_problem(21)
    na = np.full(5, na_all, dtype=np.int32)
    _, hf = oracle.gdn_verify_fold(hs, q, k, v, g, beta, na)
    for b in range(5):
        sl = slice(4 * b, 4 * b + na_all)
        _, hb = oracle.gdn_brute(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, na_all],
                                 hs[b:b + 1])
        assert rel_frob(hf[b:b + 1], hb) <= 1e-12


def test_fold_mixed_na_and_padding():
    q, k, v, g, beta, hs = _verify_problem(22)
    na = np.array([0, 4, 2, 7, 1], dtype=np.int32)  # 7: out of range -> untouched
    present = np.array([1, 1, 0, 1, 1], dtype=np.int32)
    o, hf = oracle.gdn_verify_fold(hs, q, k, v, g, beta, na, present)
    np.testing.assert_array_equal(hf[0], hs[0])
    np.testing.assert_array_equal(hf[2], hs[2])
    np.testing.assert_array_equal(hf[3], hs[3])
    assert np.all(o[8:12] == 0.0)
    assert rel_frob(hf[1], oracle.gdn_token(q[4:8], k[4:8], v[4:8], g[4:8], beta[4:8],
                                            [0, 4], hs[1:2])[1][0]) <= 1e-12


# --------------------------------------------------------------------------
# BA gates
# --------------------------------------------------------------------------

def _slot(n, vpg):
    """Slot of BA output n in the [gate | beta] row, as "ssm_ba_gates_hopper.rs"
    (ba_gates_slot) defines it: ('beta', vh) or ('gate', vh)."""
    group_dim = 2 * vpg
    within, grp = n % group_dim, n // group_dim
    if within < vpg:
        return ("beta", grp * vpg + within)
    return ("gate", grp * vpg + within - vpg)


def test_ba_slot_table_matches_golden():
    """The page's ba_gates_slot at nv = 6, vpg = 3 (tests/golden/ba_gates_slot_nv6_vpg3.txt)."""
    rows = []
    with open(os.path.join(GOLDEN, "ba_gates_slot_nv6_vpg3.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                n, kind, vh = line.split()
                rows.append((int(n), kind, int(vh)))
    assert len(rows) == 12
    for n, kind, vh in rows:
        assert _slot(n, 3) == (kind, vh)


@pytest.mark.parametrize("nv,vpg", [(48, 3), (6, 3), (8, 2), (4, 4), (5, 1)])
def test_ba_slot_is_a_bijection(nv, vpg):
    seen = {_slot(n, vpg) for n in range(2 * nv)}
    assert seen == {(kind, vh) for kind in ("gate", "beta") for vh in range(nv)}


def test_ba_gates_against_library_routines():
    rng = np.random.default_rng(30)
    M, K, nv, vpg = 23, 72, 6, 3
    x = rng.standard_normal((M, K))
    w = rng.standard_normal((2 * nv, K)) * 0.3
    a_log = rng.uniform(-1, 1, nv)
    dt_bias = rng.standard_normal(nv) * 0.1
    out = oracle.ba_gates(x, w, a_log, dt_bias, vpg)
    ba = x @ w.T
    for n in range(2 * nv):
        kind, vh = _slot(n, vpg)
        if kind == "beta":
            np.testing.assert_allclose(out[:, nv + vh], scipy.special.expit(ba[:, n]), rtol=1e-13)
        else:
            sp = np.logaddexp(0.0, ba[:, n] + dt_bias[vh])
            np.testing.assert_allclose(out[:, vh], -np.exp(a_log[vh]) * sp, rtol=1e-12)


def test_ba_gates_zero_weight():
    """W = 0: gate = -exp(A_log) softplus(dt_bias) = -exp(A_log) log(1 + e^dt), beta = 1/2."""
    M, K, nv = 3, 16, 4
    a_log = np.array([-1.0, 0.0, 0.5, 1.0])
    dt_bias = np.array([0.0, 0.1, -0.2, 3.0])
    out = oracle.ba_gates(np.ones((M, K)), np.zeros((2 * nv, K)), a_log, dt_bias, 2)
    np.testing.assert_allclose(out[:, :nv], np.broadcast_to(
        -np.exp(a_log) * np.log1p(np.exp(dt_bias)), (M, nv)), rtol=1e-14)
    np.testing.assert_array_equal(out[:, nv:], 0.5)


def test_ba_softplus_extremes():
    """Large |z|: softplus(z) -> z for z >> 0 and -> e^z for z << 0, no overflow."""
    K = 8
    x = np.ones((1, K))
    w = np.zeros((2, K))
    w[1, :] = 100.0  # gate input 800
    out = oracle.ba_gates(x, w, np.array([0.0]), np.array([0.0]), 1)
    assert out[0, 0] == pytest.approx(-800.0, rel=1e-15)
    w[1, :] = -100.0
    out = oracle.ba_gates(x, w, np.array([0.0]), np.array([0.0]), 1)
    assert out[0, 0] == pytest.approx(-np.exp(-800.0), rel=1e-12) or out[0, 0] == 0.0
