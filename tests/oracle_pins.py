"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch. tests/test_oracle_pins.py runs them on the real oracle, and
tests/test_oracle_mutants.py runs them on deliberately broken copies of the
oracle source to show that a plausible mistake fails at least one pin.

What pins what:
  hand fixture (tests/golden/hand_d2_n2.txt) -> forward, recurrence, backward, decode
  exact rational brute force (fractions)     -> forward O and state, recurrence, rows
  exact perturbation derivative (fractions)  -> backward
  lam = 1 cumulative sum (integers, exact)   -> forward, recurrence
  all-ones geometric sum closed form         -> forward, recurrence, rows
  lam -> 0 diagonal-only limit               -> forward
  time reversal                               -> reverse recurrence
  decode chain == last rows of the prefill   -> decode
  <dO,O> = <dQ,Q> = <dK,K> = <dV,V>           -> backward
  varlen == per-sequence calls               -> forward_varlen, recurrence_varlen
  exact prefix folded into the state         -> forward / recurrence with state_in
  cutting a sequence and carrying the state  -> forward / recurrence with state_in
  all-ones closed form with a constant state -> forward with state_in
  varlen with states == per-sequence calls   -> forward_varlen with state_in
  hand fixture (tests/golden/norm_gate_hand.txt) -> norm_gate (axis, layout, gate)
  constant rows closed form                  -> norm_gate (eps)
  unit rms after the norm                    -> norm_gate (the mean over H*d)
  scale invariance                           -> norm_gate
  chunk states combine to the prefix's state -> state_prefix
  exact rational chunks                      -> state_prefix
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


# ---------------------------------------------------------------- exact helpers

def _frac_forward(q, k, v, lam):
    """Exact O and state of one head by the definition, in rationals."""
    N, d = len(q), len(q[0])
    O = [[Fraction(0)] * d for _ in range(N)]
    for i in range(N):
        for j in range(i + 1):
            w = lam ** (i - j) * sum(Fraction(q[i][c]) * k[j][c] for c in range(d))
            for c in range(d):
                O[i][c] += w * v[j][c]
    S = [[Fraction(0)] * d for _ in range(d)]
    for j in range(N):
        w = lam ** (N - 1 - j)
        for a in range(d):
            for b in range(d):
                S[a][b] += w * k[j][a] * v[j][b]
    return O, S


def _frac_objective(dout, q, k, v, lam):
    O, _ = _frac_forward(q, k, v, lam)
    return sum(Fraction(dout[i][c]) * O[i][c] for i in range(len(O)) for c in range(len(O[0])))


def _as_frac(a):
    return [[Fraction(float(x)) for x in row] for row in a]


def _rand_int(rng, shape, lo=-3, hi=3):
    return rng.integers(lo, hi + 1, size=shape).astype(np.float64)


# ---------------------------------------------------------------- pins

def pin_hand_fixture(orc):
    g = _read_golden("hand_d2_n2.txt")
    lam = np.array([g["lam"][0]])
    q, k, v, do = (g[x].reshape(1, 1, 2, 2) for x in ("q", "k", "v", "dO"))
    o, st = orc.forward(q, k, v, lam)
    assert np.array_equal(o.reshape(-1), g["O"]), (o, g["O"])
    assert np.array_equal(st.reshape(-1), g["state"]), (st, g["state"])
    o2, st2 = orc.recurrence(q, k, v, lam)
    assert np.array_equal(o2.reshape(-1), g["O"])
    assert np.array_equal(st2.reshape(-1), g["state"])
    dq, dk, dv = orc.backward(do, q, k, v, lam)
    assert np.array_equal(dq.reshape(-1), g["dQ"]), dq
    assert np.array_equal(dk.reshape(-1), g["dK"]), dk
    assert np.array_equal(dv.reshape(-1), g["dV"]), dv
    od, sd = orc.decode(g["dec_q"].reshape(1, 1, 2), g["dec_k"].reshape(1, 1, 2),
                        g["dec_v"].reshape(1, 1, 2), lam, st)
    assert np.array_equal(sd.reshape(-1), g["dec_state"]), sd
    assert np.array_equal(od.reshape(-1), g["dec_o"]), od


def pin_rational_brute_force(orc, seed=0):
    rng = np.random.default_rng(seed)
    lam = Fraction(1, 2)
    for (N, d) in ((1, 1), (5, 2), (9, 3), (12, 4)):
        q, k, v = (_rand_int(rng, (N, d)) for _ in range(3))
        O, S = _frac_forward(_as_frac(q), _as_frac(k), _as_frac(v), lam)
        O = np.array([[float(x) for x in r] for r in O])
        S = np.array([[float(x) for x in r] for r in S])
        args = [x.reshape(1, 1, N, d) for x in (q, k, v)]
        o1, s1 = orc.forward(*args, np.array([0.5]))
        assert np.array_equal(o1[0, 0], O) and np.array_equal(s1[0, 0], S), (N, d)
        o2, s2 = orc.recurrence(*args, np.array([0.5]))
        assert np.array_equal(o2[0, 0], O) and np.array_equal(s2[0, 0], S), (N, d)
        rows = np.arange(N)[::-1].copy()
        o3 = orc.forward_rows(q, k, v, 0.5, rows)
        assert np.array_equal(o3, O[rows]), (N, d)


def pin_backward_exact_perturbation(orc, seed=1):
    """f(X) = <dO, O(Q,K,V)> is linear in each of Q, K, V alone, so
    f(X + e) - f(X) is the exact partial derivative along unit vector e."""
    rng = np.random.default_rng(seed)
    lam = Fraction(1, 2)
    N, d = 5, 2
    q, k, v, do = (_rand_int(rng, (N, d)) for _ in range(4))
    Fq, Fk, Fv, Fdo = (_as_frac(x) for x in (q, k, v, do))
    f0 = _frac_objective(Fdo, Fq, Fk, Fv, lam)
    grads = []
    for which in range(3):
        G = np.zeros((N, d))
        for i in range(N):
            for c in range(d):
                X = [[Fraction(x) for x in row] for row in (Fq, Fk, Fv)[which]]
                X[i][c] += 1
                ops = [Fq, Fk, Fv]
                ops[which] = X
                G[i, c] = float(_frac_objective(Fdo, *ops, lam) - f0)
        grads.append(G)
    dq, dk, dv = orc.backward(*(x.reshape(1, 1, N, d) for x in (do, q, k, v)), np.array([0.5]))
    for got, want, name in zip((dq, dk, dv), grads, "QKV"):
        assert np.array_equal(got[0, 0], want), (name, got[0, 0], want)


def pin_lambda_one_cumsum(orc, seed=2):
    """lam = 1: O_i = q_i (sum_{j<=i} k_j^T v_j), state = K^T V (exact on integers)."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 2, 2, 37, 6
    q, k, v = (_rand_int(rng, (B, H, N, d)) for _ in range(3))
    prefix = np.cumsum(np.einsum("bhna,bhnc->bhnac", k, v), axis=2)
    want_o = np.einsum("bhna,bhnac->bhnc", q, prefix)
    want_s = np.einsum("bhna,bhnc->bhac", k, v)
    lam = np.ones(H)
    for fn in (orc.forward, orc.recurrence):
        o, s = fn(q, k, v, lam)
        assert np.array_equal(o, want_o) and np.array_equal(s, want_s)


def pin_all_ones_geometric(orc):
    """q = k = v = 1: O_i[c] = d (1 - lam^(i+1)) / (1 - lam), state = (1 - lam^N)/(1 - lam)."""
    N, d = 300, 8
    lam = np.array([0.3, 0.9, 0.999])
    ones = np.ones((1, 3, N, d))
    i = np.arange(N)[None, :, None]
    l = lam[:, None, None]
    want_o = d * (1 - l ** (i + 1)) / (1 - l) * np.ones((3, N, d))
    want_s = ((1 - lam ** N) / (1 - lam))[:, None, None] * np.ones((3, d, d))
    for fn in (orc.forward, orc.recurrence):
        o, s = fn(ones, ones, ones, lam)
        np.testing.assert_allclose(o[0], want_o, rtol=1e-12)
        np.testing.assert_allclose(s[0], want_s, rtol=1e-12)
    rows = np.array([0, 1, 255, 256, 299])
    got = orc.forward_rows(ones[0, 2], ones[0, 2], ones[0, 2], lam[2], rows)
    np.testing.assert_allclose(got, want_o[2][rows], rtol=1e-12)


def pin_lambda_zero_diagonal(orc, seed=3):
    """lam -> 0: O_i -> (q_i . k_i) v_i, state -> k_{N-1}^T v_{N-1}."""
    rng = np.random.default_rng(seed)
    N, d = 40, 5
    q, k, v = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    lam = np.array([np.exp(-60.0)])
    o, s = orc.forward(q, k, v, lam)
    want = np.einsum("na,na->n", q[0, 0], k[0, 0])[:, None] * v[0, 0]
    # the neglected terms are ~1e-26 relative; only fp64 rounding remains
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], np.outer(k[0, 0, -1], v[0, 0, -1]), rtol=1e-14,
                               atol=1e-14)


def pin_recurrence_matches_quadratic(orc, seed=4):
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 3, 150, 16
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.4, 0.95, 0.9961])
    o1, s1 = orc.forward(q, k, v, lam)
    o2, s2 = orc.recurrence(q, k, v, lam)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12 * np.abs(o1).max())
    np.testing.assert_allclose(s2, s1, rtol=1e-11, atol=1e-12 * np.abs(s1).max())


def pin_reverse_is_time_reversal(orc, seed=5):
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 2, 33, 4
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.7, 0.99])
    flip = lambda x: x[:, :, ::-1].copy()
    o_r, s_r = orc.recurrence(q, k, v, lam, reverse=True)
    o_f, s_f = orc.forward(flip(q), flip(k), flip(v), lam)
    np.testing.assert_allclose(o_r, flip(o_f), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s_r, s_f, rtol=1e-12, atol=1e-13)


def pin_decode_chain(orc, seed=6):
    """prefill(N - m) state followed by m decode steps reproduces the last m rows
    and the final state of prefill(N)."""
    rng = np.random.default_rng(seed)
    B, H, N, d, m = 2, 2, 20, 6, 5
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.6, 0.97])
    o_full, s_full = orc.forward(q, k, v, lam)
    _, st = orc.forward(q[:, :, :N - m], k[:, :, :N - m], v[:, :, :N - m], lam)
    for t in range(N - m, N):
        o_t, st = orc.decode(q[:, :, t], k[:, :, t], v[:, :, t], lam, st)
        np.testing.assert_allclose(o_t, o_full[:, :, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st, s_full, rtol=1e-12, atol=1e-12)


def pin_backward_identities(orc, seed=7):
    """O is degree-1 homogeneous in each of Q, K, V, so by Euler's identity
    <dO, O> = <dQ, Q> = <dK, K> = <dV, V>; the recurrence form of the gradients
    agrees with the quadratic sums."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 2, 45, 8
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    lam = np.array([0.8, 0.995])
    o, _ = orc.forward(q, k, v, lam)
    dq, dk, dv = orc.backward(do, q, k, v, lam)
    ref = np.sum(do * o)
    for g, x in ((dq, q), (dk, k), (dv, v)):
        np.testing.assert_allclose(np.sum(g * x), ref, rtol=1e-11)
    for g1, g2 in zip((dq, dk, dv), orc.backward_recurrence(do, q, k, v, lam)):
        np.testing.assert_allclose(g2, g1, rtol=1e-10, atol=1e-12 * np.abs(g1).max())


def pin_varlen_is_per_sequence(orc, seed=8):
    rng = np.random.default_rng(seed)
    H, d = 2, 4
    lengths = [7, 0, 1, 13, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q, k, v = (rng.standard_normal((H, T, d)) for _ in range(3))
    lam = np.array([0.5, 0.9])
    for fn, seq_fn in ((orc.forward_varlen, orc.forward),
                       (orc.recurrence_varlen, orc.recurrence)):
        o, st = fn(cu, q, k, v, lam)
        for s, L in enumerate(lengths):
            a, b = cu[s], cu[s + 1]
            if L == 0:
                assert np.all(st[s] == 0)
                continue
            o_s, st_s = seq_fn(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b], lam)
            np.testing.assert_allclose(o[:, a:b], o_s[0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(st[s], st_s[0], rtol=1e-13, atol=1e-14)


def _floats(rows, shape):
    return np.array([[float(x) for x in r] for r in rows], dtype=np.float64).reshape(shape)


def pin_state_in_exact_prefix(orc, seed=9):
    """A prefix of m tokens folded into S_in (its exact state) and the n tokens
    after it reproduce the exact rows and final state of the whole sequence
    (lam = 1/2 and small integers: every value is exact in fp64)."""
    rng = np.random.default_rng(seed)
    lam = Fraction(1, 2)
    for (m, n, d) in ((1, 1, 1), (3, 4, 2), (4, 7, 3), (5, 0, 2), (2, 6, 4)):
        N = m + n
        q, k, v = (_rand_int(rng, (N, d)) for _ in range(3))
        O, S = _frac_forward(_as_frac(q), _as_frac(k), _as_frac(v), lam)
        _, Sp = _frac_forward(_as_frac(q[:m]), _as_frac(k[:m]), _as_frac(v[:m]), lam)
        s_in = _floats(Sp, (1, 1, d, d))
        args = [x[m:].reshape(1, 1, n, d) for x in (q, k, v)]
        want_o, want_s = _floats(O[m:], (n, d)), _floats(S, (d, d))
        for fn in (orc.forward, orc.recurrence):
            o, st = fn(*args, np.array([0.5]), state_in=s_in)
            assert np.array_equal(o[0, 0], want_o), (fn.__name__, m, n, d, o[0, 0], want_o)
            assert np.array_equal(st[0, 0], want_s), (fn.__name__, m, n, d, st[0, 0], want_s)


def pin_state_in_split_invariance(orc, seed=10):
    """Cutting a sequence at any m and carrying the state across the cut gives
    rows m.. and the final state of the uncut sequence."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 2, 3, 60, 6
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.45, 0.9, 0.999])
    o_full, s_full = orc.forward(q, k, v, lam)
    to = 1e-12 * np.abs(o_full).max()
    ts = 1e-12 * np.abs(s_full).max()
    for m in (0, 1, 17, 59, 60):
        _, s_m = orc.forward(q[:, :, :m], k[:, :, :m], v[:, :, :m], lam)
        tail = [x[:, :, m:] for x in (q, k, v)]
        for fn in (orc.forward, orc.recurrence):
            o2, s2 = fn(*tail, lam, state_in=s_m)
            np.testing.assert_allclose(o2, o_full[:, :, m:], rtol=1e-11, atol=to)
            np.testing.assert_allclose(s2, s_full, rtol=1e-11, atol=ts)


def pin_state_in_all_ones(orc):
    """q = k = v = 1 and S_in = c in every entry:
    O_i[b] = lam^(i+1) d c + d (1 - lam^(i+1)) / (1 - lam),
    state  = lam^N c + (1 - lam^N) / (1 - lam)."""
    N, d, c = 200, 8, 2.5
    lam = np.array([0.3, 0.9, 0.999])
    ones = np.ones((1, 3, N, d))
    s_in = np.full((1, 3, d, d), c)
    i = np.arange(N)[None, :, None]
    l = lam[:, None, None]
    want_o = (l ** (i + 1) * d * c + d * (1 - l ** (i + 1)) / (1 - l)) * np.ones((3, N, d))
    want_s = (lam ** N * c + (1 - lam ** N) / (1 - lam))[:, None, None] * np.ones((3, d, d))
    o, s = orc.forward(ones, ones, ones, lam, state_in=s_in)
    np.testing.assert_allclose(o[0], want_o, rtol=1e-12)
    np.testing.assert_allclose(s[0], want_s, rtol=1e-12)


def pin_state_in_varlen_is_per_sequence(orc, seed=11):
    rng = np.random.default_rng(seed)
    H, d = 2, 4
    lengths = [5, 0, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q, k, v = (rng.standard_normal((H, T, d)) for _ in range(3))
    s_in = rng.standard_normal((len(lengths), H, d, d))
    lam = np.array([0.5, 0.9])
    for fn, seq_fn in ((orc.forward_varlen, orc.forward),
                       (orc.recurrence_varlen, orc.recurrence)):
        o, st = fn(cu, q, k, v, lam, state_in=s_in)
        for s, L in enumerate(lengths):
            a, b = cu[s], cu[s + 1]
            if L == 0:
                assert np.array_equal(st[s], s_in[s])
                continue
            o_s, st_s = seq_fn(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b], lam,
                               state_in=s_in[s][None])
            np.testing.assert_allclose(o[:, a:b], o_s[0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(st[s], st_s[0], rtol=1e-13, atol=1e-14)


def pin_norm_gate_hand_fixture(orc):
    path = os.path.join(GOLDEN, "norm_gate_hand.txt")
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            g3 = np.log(3.0)
            vals[key] = np.array([g3 if x == "g3" else -g3 if x == "-g3" else float(x)
                                  for x in nums])
    y = orc.norm_gate(vals["O"].reshape(1, 2, 2, 2), vals["G"].reshape(1, 2, 4), vals["w"],
                      float(vals["eps"][0]))
    np.testing.assert_allclose(y.reshape(-1), vals["Y"], rtol=1e-14, atol=0)


def pin_norm_gate_constant_rows(orc):
    """O = c everywhere, G = 0, w = 1: Y = c / sqrt(c^2 + eps) / 2."""
    B, H, N, d, c, eps = 2, 3, 5, 4, 3.0, 0.25
    o = np.full((B, H, N, d), c)
    y = orc.norm_gate(o, np.zeros((B, N, H * d)), np.ones(H * d), eps)
    np.testing.assert_allclose(y, np.full((B, N, H * d), c / np.sqrt(c * c + eps) / 2),
                               rtol=1e-14)


def pin_norm_gate_unit_rms(orc, seed=12):
    """eps = 0, w = 1 and a saturated gate: every token's Y has mean square 1
    over its H*d features."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 2, 4, 7, 8
    o = rng.standard_normal((B, H, N, d)) * rng.uniform(0.1, 10, size=(B, H, N, 1))
    y = orc.norm_gate(o, np.full((B, N, H * d), 50.0), np.ones(H * d), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=2), 1.0, rtol=1e-13)


def pin_norm_gate_scale_invariance(orc, seed=13):
    """Y(a O, a^2 eps) = Y(O, eps)."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 3, 6, 4
    o = rng.standard_normal((B, H, N, d))
    g = rng.standard_normal((B, N, H * d))
    w = rng.standard_normal(H * d)
    a, eps = 7.25, 0.3
    np.testing.assert_allclose(orc.norm_gate(a * o, g, w, a * a * eps),
                               orc.norm_gate(o, g, w, eps), rtol=1e-13, atol=1e-15)


def pin_state_prefix_split(orc, seed=14):
    """Cut a sequence into chunks of unequal length: combining the chunks'
    local states gives, for every r, the state of chunks 0..r-1 taken as one
    sequence (the quadratic form over the concatenation)."""
    rng = np.random.default_rng(seed)
    B, H, d = 1, 3, 5
    lens = [7, 1, 0, 12, 4]
    N = sum(lens)
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.5, 0.9, 0.999])
    cuts = np.concatenate([[0], np.cumsum(lens)])
    states = np.stack([orc.forward(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], lam)[1]
                       for a, b in zip(cuts[:-1], cuts[1:])])
    for r in range(len(lens) + 1):
        got = orc.state_prefix(states, lam, lens, r)
        _, want = orc.forward(q[:, :, :cuts[r]], k[:, :, :cuts[r]], v[:, :, :cuts[r]], lam)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def pin_state_prefix_exact(orc):
    """lam = 1/2 and small integer chunk states: S_in(3) = lam^(n1+n2) S0 +
    lam^n2 S1 + S2 exactly, written out for three chunks."""
    S = np.arange(3 * 4, dtype=np.float64).reshape(3, 1, 1, 2, 2) - 5
    lens = [3, 2, 1]
    got = orc.state_prefix(S, np.array([0.5]), lens, 3)[0, 0]
    want = 0.5 ** 3 * S[0, 0, 0] + 0.5 ** 1 * S[1, 0, 0] + S[2, 0, 0]
    assert np.array_equal(got, want), (got, want)
    assert np.array_equal(orc.state_prefix(S, np.array([0.5]), lens, 0)[0, 0], np.zeros((2, 2)))


ALL_PINS = [
    pin_hand_fixture,
    pin_rational_brute_force,
    pin_backward_exact_perturbation,
    pin_lambda_one_cumsum,
    pin_all_ones_geometric,
    pin_lambda_zero_diagonal,
    pin_recurrence_matches_quadratic,
    pin_reverse_is_time_reversal,
    pin_decode_chain,
    pin_backward_identities,
    pin_varlen_is_per_sequence,
    pin_state_in_exact_prefix,
    pin_state_in_split_invariance,
    pin_state_in_all_ones,
    pin_state_in_varlen_is_per_sequence,
    pin_norm_gate_hand_fixture,
    pin_norm_gate_constant_rows,
    pin_norm_gate_unit_rms,
    pin_norm_gate_scale_invariance,
    pin_state_prefix_split,
    pin_state_prefix_exact,
]
