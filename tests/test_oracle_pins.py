"""Pins of the fp64 oracle against what the mathematics of the gated delta rule fixes.

Recurrence (published gated delta rule; the state recurrence behind the Ferrite project page,
Design section 03 "Chunked Gated DeltaNet"):
    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t / sqrt(dk)

Each test checks the oracle against something other than itself: hand-worked values, closed forms,
invariants, special cases that reduce to textbook rules, an explicit-matrix expansion, and the
chunkwise WY/UT form (a different algebraic route to the same result).  The plausible mistakes each
one catches are noted beside it.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_d2.txt")


def rnd(T, H, dk, dv, seed, gate=(-0.5, 0.0), normalise=True, N=None):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, H, dk))
    k = r.standard_normal((T, H, dk))
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, H, dv))
    g = r.uniform(gate[0], gate[1], (T, H))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    s0 = None if N is None else 0.05 * r.standard_normal((N, H, dv, dk))
    return q, k, v, g, beta, s0


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------------------------------------
# hand-worked values (tests/golden/hand_d2.txt)
# ---------------------------------------------------------------------------------------------
def _parse_golden():
    cases, cur = {}, None
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "case":
            cur = cases.setdefault(tok[1], dict(S0=None, tokens=[], o=[], S=None))
        elif tok[0] == "S0":
            cur["S0"] = np.array(tok[1:], float).reshape(2, 2)
        elif tok[0] == "token":
            d = {}
            i = 1
            while i < len(tok):
                key = tok[i]
                n = 2 if key in ("q", "k", "v") else 1
                d[key] = np.array(tok[i + 1:i + 1 + n], float)
                i += 1 + n
            cur["tokens"].append(d)
        elif tok[0] == "o":
            cur["o"].append(np.array(tok[1:], float))
        elif tok[0] == "S":
            cur["S"] = np.array(tok[1:], float).reshape(2, 2)
    return cases


@pytest.mark.parametrize("case", ["A", "B"])
def test_hand_worked_golden(case):
    c = _parse_golden()[case]
    T = len(c["tokens"])
    q = np.array([t["q"] for t in c["tokens"]])[:, None, :]
    k = np.array([t["k"] for t in c["tokens"]])[:, None, :]
    v = np.array([t["v"] for t in c["tokens"]])[:, None, :]
    g = np.log(np.array([t["alpha"][0] for t in c["tokens"]]))[:, None]
    b = np.array([t["beta"][0] for t in c["tokens"]])[:, None]
    o, s = oracle.recurrence(q, k, v, g, b, state_in=c["S0"][None, None])
    np.testing.assert_allclose(o[:, 0, :] * np.sqrt(2.0), np.array(c["o"]), atol=1e-13)
    np.testing.assert_allclose(s[0, 0], c["S"], atol=1e-13)
    # the chunked form and the brute-force expansion reproduce the same hand values
    for C in (1, 2, 3):
        oc, sc = oracle.chunked(q, k, v, g, b, C, state_in=c["S0"][None, None])
        np.testing.assert_allclose(oc[:, 0, :] * np.sqrt(2.0), np.array(c["o"]), atol=1e-13)
        np.testing.assert_allclose(sc[0, 0], c["S"], atol=1e-13)
    ob, sb = oracle.brute_force(q, k, v, g, b, state_in=c["S0"][None, None])
    np.testing.assert_allclose(ob[:, 0, :] * np.sqrt(2.0), np.array(c["o"]), atol=1e-13)
    assert T == len(c["o"])


# ---------------------------------------------------------------------------------------------
# brute-force expansion with explicit matrices (catches a wrong operand order, a transposed
# product, a gate applied to the write term, a missing scale)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,dk,dv,seed", [(1, 4, 4, 0), (5, 6, 3, 1), (8, 8, 8, 2), (7, 3, 5, 3)])
def test_brute_force_expansion(T, dk, dv, seed):
    q, k, v, g, b, s0 = rnd(T, 2, dk, dv, seed, N=1)
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    ob, sb = oracle.brute_force(q, k, v, g, b, state_in=s0)
    assert rel(o, ob) < 1e-12 and rel(s, sb) < 1e-12


# ---------------------------------------------------------------------------------------------
# special cases with closed forms
# ---------------------------------------------------------------------------------------------
def test_beta0_gate0_state_unchanged():
    """beta = 0 and g = 0: S never changes, o_t = S_0 q_t / sqrt(dk)."""
    q, k, v, g, b, s0 = rnd(40, 3, 16, 12, 4, N=1)
    g[:] = 0.0
    b[:] = 0.0
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    np.testing.assert_array_equal(s, s0)
    expect = np.einsum("hrc,thc->thr", s0[0], q) / 4.0
    assert rel(o, expect) < 1e-13


def test_beta0_pure_decay():
    """beta = 0: S_t = exp(g_1 + ... + g_t) S_0 (closed form of the decay)."""
    q, k, v, g, b, s0 = rnd(25, 2, 8, 8, 5, N=1)
    b[:] = 0.0
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    decay = np.exp(g.sum(axis=0))                 # [H]
    assert rel(s[0], decay[:, None, None] * s0[0]) < 1e-13
    cum = np.exp(np.cumsum(g, axis=0))            # [T, H]
    expect = cum[:, :, None] * np.einsum("hrc,thc->thr", s0[0], q) / np.sqrt(8)
    assert rel(o, expect) < 1e-12


def test_gate0_is_textbook_delta_rule():
    """g = 0 reduces to the (ungated) delta rule in its Widrow-Hoff form
    S <- S + beta (v - S k) k^T (Schlag et al. 2021; Yang et al. 2024, "Parallelizing Linear
    Transformers with the Delta Rule over Sequence Length")."""
    T, H, dk, dv = 30, 2, 10, 7
    q, k, v, g, b, s0 = rnd(T, H, dk, dv, 6, N=1)
    g[:] = 0.0
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    for h in range(H):
        S = s0[0, h].copy()
        for t in range(T):
            err = v[t, h] - S @ k[t, h]
            S = S + b[t, h] * np.outer(err, k[t, h])
            assert rel(o[t, h], S @ q[t, h] / np.sqrt(dk)) < 1e-12
        assert rel(s[0, h], S) < 1e-12


def test_beta1_unit_key_writes_value_exactly():
    """beta = 1 with a unit key: S_t k_t = v_t for any gate and any history
    (alpha S (I - k k^T) k = 0, v k^T k = v).  Catches the gate multiplying the write term and a
    sign error in the projection."""
    q, k, v, g, b, s0 = rnd(20, 3, 12, 9, 7, N=1)
    b[:] = 1.0
    for t in range(1, 21):
        _, s = oracle.recurrence(q[:t], k[:t], v[:t], g[:t], b[:t], state_in=s0)
        sk = np.einsum("hrc,hc->hr", s[0], k[t - 1])
        assert np.max(np.abs(sk - v[t - 1])) < 1e-13


def test_orthonormal_keys_associative_memory():
    """alpha = 1, beta = 1, S_0 = 0 and orthonormal keys: S = sum_j v_j k_j^T, and o_t reads back
    v_j for q_t = k_j (j <= t)."""
    dk = dv = 8
    T = 8
    r = np.random.default_rng(8)
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    k = Qm.T[:, None, :].copy()                  # T orthonormal keys
    v = r.standard_normal((T, 1, dv))
    g = np.zeros((T, 1))
    b = np.ones((T, 1))
    q = k[::-1].copy()                           # q_t = k_{T-1-t}
    o, s = oracle.recurrence(q, k, v, g, b)
    assert rel(s[0, 0], sum(np.outer(v[j, 0], k[j, 0]) for j in range(T))) < 1e-13
    for t in range(T):
        j = T - 1 - t
        expect = v[j, 0] / np.sqrt(dk) if j <= t else np.zeros(dv)
        assert np.max(np.abs(o[t, 0] - expect)) < 1e-12


def test_linearity_in_values_and_state():
    """(V, S_0) -> (c V, c S_0) scales o and S by c (the recurrence is linear in them)."""
    q, k, v, g, b, s0 = rnd(33, 2, 6, 5, 9, N=1)
    o1, s1 = oracle.recurrence(q, k, v, g, b, state_in=s0)
    o2, s2 = oracle.recurrence(q, k, -2.5 * v, g, b, state_in=-2.5 * s0)
    assert rel(o2, -2.5 * o1) < 1e-13 and rel(s2, -2.5 * s1) < 1e-13


# ---------------------------------------------------------------------------------------------
# the chunkwise WY/UT form (a different route through the algebra) against the recurrence
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 4, 8, 32, 64])
def test_chunk_size_invariance(C):
    lengths = [75, 32, 1, 64, 13]
    cu = np.cumsum([0] + lengths)
    q, k, v, g, b, s0 = rnd(int(cu[-1]), 2, 16, 8, 10, N=len(lengths))
    o, s = oracle.recurrence(q, k, v, g, b, cu_seqlens=cu, state_in=s0)
    oc, sc = oracle.chunked(q, k, v, g, b, C, cu_seqlens=cu, state_in=s0)
    assert rel(oc, o) < 1e-12 and rel(sc, s) < 1e-12


def test_chunked_strong_decay_and_large_beta():
    """Strong gates (g down to -8 per token) stress exp(gamma_i - gamma_j) inside a chunk."""
    q, k, v, g, b, s0 = rnd(96, 2, 16, 16, 11, gate=(-8.0, 0.0), N=1)
    b[:] = 0.999
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    oc, sc = oracle.chunked(q, k, v, g, b, 32, state_in=s0)
    assert rel(oc, o) < 1e-11 and rel(sc, s) < 1e-11


# ---------------------------------------------------------------------------------------------
# state carry, packing and causality (Ferrite page, Design section 07: a resumed prompt equals
# one computed in full; section 06: output independent of co-running requests; "The Mask Is Not
# the Model": prefix invariance across chunk boundaries)
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("cut", [1, 31, 32, 33, 70])
def test_split_sequence_equivalence(cut):
    q, k, v, g, b, s0 = rnd(100, 2, 12, 10, 12, N=1)
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0)
    oa, sa = oracle.recurrence(q[:cut], k[:cut], v[:cut], g[:cut], b[:cut], state_in=s0)
    ob, sb = oracle.recurrence(q[cut:], k[cut:], v[cut:], g[cut:], b[cut:], state_in=sa)
    np.testing.assert_array_equal(np.concatenate([oa, ob]), o)
    np.testing.assert_array_equal(sb, s)


def test_packing_equals_separate_calls():
    lengths = [17, 0, 40, 3]
    cu = np.cumsum([0] + lengths)
    q, k, v, g, b, s0 = rnd(int(cu[-1]), 2, 8, 8, 13, N=len(lengths))
    o, s = oracle.recurrence(q, k, v, g, b, cu_seqlens=cu, state_in=s0)
    for n in range(len(lengths)):
        a, e = cu[n], cu[n + 1]
        on, sn = oracle.recurrence(q[a:e], k[a:e], v[a:e], g[a:e], b[a:e], state_in=s0[n:n + 1])
        np.testing.assert_array_equal(o[a:e], on)
        np.testing.assert_array_equal(s[n], sn[0])
    np.testing.assert_array_equal(s[1], s0[1])   # a zero-length sequence keeps its state


@pytest.mark.parametrize("t", [0, 31, 32, 63, 64, 90])
def test_prefix_invariance(t):
    q, k, v, g, b, s0 = rnd(128, 2, 8, 8, 14, N=1)
    o, _ = oracle.recurrence(q, k, v, g, b, state_in=s0)
    q2, k2, v2, g2, b2 = (x.copy() for x in (q, k, v, g, b))
    r = np.random.default_rng(99)
    for x in (q2, k2, v2):
        x[t + 1:] += r.standard_normal(x[t + 1:].shape)
    g2[t + 1:] = -r.uniform(0, 1, g2[t + 1:].shape)
    b2[t + 1:] = r.uniform(0, 1, b2[t + 1:].shape)
    o2, _ = oracle.recurrence(q2, k2, v2, g2, b2, state_in=s0)
    oc, _ = oracle.chunked(q2, k2, v2, g2, b2, 32, state_in=s0)
    np.testing.assert_array_equal(o2[:t + 1], o[:t + 1])
    assert rel(oc[:t + 1], o[:t + 1]) < 1e-12
    assert np.max(np.abs(o2[t + 1:] - o[t + 1:])) > 1e-3   # the perturbation did reach the future


def test_rows_match_full_recurrence():
    lengths = [50, 9, 70]
    cu = np.cumsum([0] + lengths)
    q, k, v, g, b, s0 = rnd(int(cu[-1]), 3, 8, 6, 15, N=3)
    o, s = oracle.recurrence(q, k, v, g, b, cu_seqlens=cu, state_in=s0)
    samples = np.array([[0, 0, 0], [1, 2, 5], [2, 1, 3], [2, 2, 0]])
    orow, srow = oracle.rows(q, k, v, g, b, samples, cu_seqlens=cu, state_in=s0)
    for i, (n, h, r) in enumerate(samples):
        a, e = cu[n], cu[n + 1]
        np.testing.assert_allclose(orow[i, a:e], o[a:e, h, r], rtol=0, atol=1e-14)
        assert np.all(np.isnan(orow[i, :a])) and np.all(np.isnan(orow[i, e:]))
        np.testing.assert_allclose(srow[i], s[n, h, r], rtol=0, atol=1e-14)


def test_decode_step_is_length_one_recurrence():
    B, H, d = 5, 2, 8
    q, k, v, g, b, s0 = rnd(B, H, d, d, 16, N=B)
    o, s = oracle.decode_step(q, k, v, g, b, s0)
    for i in range(B):
        S = s0[i]
        for h in range(H):
            a = np.exp(g[i, h])
            Sn = a * S[h] @ (np.eye(d) - b[i, h] * np.outer(k[i, h], k[i, h])) + b[i, h] * np.outer(v[i, h], k[i, h])
            assert rel(s[i, h], Sn) < 1e-13
            assert rel(o[i, h], Sn @ q[i, h] / np.sqrt(d)) < 1e-13


def test_l2norm_unit_length_direction_and_degenerate_vectors():
    r = np.random.default_rng(51)
    x = r.standard_normal((7, 3, 16)) * r.uniform(0.01, 100.0, (7, 3, 1))
    y = oracle.l2norm(x)
    assert np.max(np.abs(np.linalg.norm(y, axis=-1) - 1.0)) < 1e-14
    # same direction: y is a positive multiple of x
    cos = np.sum(x * y, axis=-1) / np.linalg.norm(x, axis=-1)
    assert np.max(np.abs(cos - 1.0)) < 1e-14
    assert rel(oracle.l2norm(3.5 * x), y) < 1e-15               # scale invariance
    assert rel(oracle.l2norm(y), y) < 1e-15                     # idempotent
    z = np.zeros((2, 5))
    assert np.array_equal(oracle.l2norm(z), z)                  # zero vector stays zero
    tiny = np.full((1, 4), 1e-14)                               # norm below eps: divided by eps
    assert rel(oracle.l2norm(tiny), tiny / 1e-12) < 1e-15


def test_states_at_cuts_equal_prefix_runs():
    """A snapshot at cut c equals the final state of the recurrence over the sequence's tokens
    before c, and cutting changes neither the outputs nor the final states."""
    q, k, v, g, b, s0 = rnd(90, 2, 6, 5, 31, N=3)
    cu = np.array([0, 40, 40, 90])
    cuts = [1, 17, 39, 41, 77]
    o, st, sn = oracle.states_at(q, k, v, g, b, cuts, cu_seqlens=cu, state_in=s0)
    o1, st1 = oracle.recurrence(q, k, v, g, b, cu_seqlens=cu, state_in=s0)
    assert rel(o, o1) < 1e-13 and rel(st, st1) < 1e-13
    for i, c in enumerate(cuts):
        n = int(np.searchsorted(cu, c, side="right")) - 1
        _, sp = oracle.recurrence(q[cu[n]:c], k[cu[n]:c], v[cu[n]:c], g[cu[n]:c], b[cu[n]:c], state_in=s0[n:n + 1])
        assert rel(sn[i], sp[0]) < 1e-13


def test_decode_verify_states_match_brute_force():
    """The state after each drafted token equals the explicit-matrix expansion over that prefix, and
    the outputs are S_t q_t / sqrt(dk); the committed state is left untouched."""
    B, Tk, H, d = 2, 5, 2, 6
    r = np.random.default_rng(21)
    q, k, v, g, b, _ = rnd(B * Tk, H, d, d, 22)
    q, k, v = (x.reshape(B, Tk, H, d) for x in (q, k, v))
    g, b = g.reshape(B, Tk, H), b.reshape(B, Tk, H)
    s0 = 0.05 * r.standard_normal((B, H, d, d))
    keep = s0.copy()
    o, st = oracle.decode_verify(q, k, v, g, b, s0)
    assert np.array_equal(s0, keep)
    for i in range(B):
        for t in range(Tk):
            ob, sb = oracle.brute_force(q[i, :t + 1], k[i, :t + 1], v[i, :t + 1], g[i, :t + 1], b[i, :t + 1],
                                        state_in=s0[i][None])
            assert rel(st[i, t], sb[0]) < 1e-12
            assert rel(o[i, t], ob[t]) < 1e-12


def test_decode_verify_equals_one_sequence_per_draft_chain():
    """Tk drafted tokens of B sequences = the recurrence over B sequences of Tk tokens each."""
    B, Tk, H, d = 3, 7, 2, 8
    q, k, v, g, b, _ = rnd(B * Tk, H, d, d, 23)
    s0 = 0.05 * np.random.default_rng(24).standard_normal((B, H, d, d))
    o, st = oracle.decode_verify(*(x.reshape((B, Tk) + x.shape[1:]) for x in (q, k, v, g, b)), s0)
    o2, s2 = oracle.recurrence(q, k, v, g, b, cu_seqlens=np.arange(0, B * Tk + 1, Tk), state_in=s0)
    assert rel(o.reshape(B * Tk, H, d), o2) < 1e-13
    assert rel(st[:, -1], s2) < 1e-13


def _one_head(L, d, seed, gate=(-0.5, 0.0)):
    q, k, v, g, b, _ = rnd(L, 1, d, d, seed, gate=gate)
    return q[:, 0], k[:, 0], v[:, 0], g[:, 0], b[:, 0]


@pytest.mark.parametrize("L", [1, 5, 31, 32])
@pytest.mark.parametrize("gate", [(-0.5, 0.0), (-4.0, -1.0)])
def test_chunk_operator_reconstructs_the_recurrence(L, gate):
    """One chunk built from the WY/UT quantities (T'', P T'', gates) gives the recurrence's outputs
    and state, for ragged chunks and strong gates."""
    d = 16
    q, k, v, g, b = _one_head(L, d, 60 + L, gate)
    S0 = 0.05 * np.random.default_rng(61).standard_normal((d, d))
    op = oracle.chunk_operator(q, k, g, b)
    O, S1 = oracle.chunk_step(op, q, k, v, S0)
    o2, s2 = oracle.recurrence(q[:, None], k[:, None], v[:, None], g[:, None], b[:, None], state_in=S0[None, None])
    assert rel(O, o2[:, 0]) < 1e-12 and rel(S1, s2[0, 0]) < 1e-12


@pytest.mark.parametrize("L", [33, 63, 64])
@pytest.mark.parametrize("gate", [(-0.5, 0.0), (-4.0, -1.0)])
def test_pair_operator_reconstructs_the_recurrence(L, gate):
    """The same over 64 rows (two chunks of 32 carried as one step): the operator over a pair of
    chunks gives the recurrence's outputs and state, the last pair of a sequence being short."""
    d = 16
    q, k, v, g, b = _one_head(L, d, 70 + L, gate)
    S0 = 0.05 * np.random.default_rng(71).standard_normal((d, d))
    op = oracle.chunk_operator(q, k, g, b, chunk=64)
    O, S1 = oracle.chunk_step(op, q, k, v, S0, chunk=64)
    o2, s2 = oracle.recurrence(q[:, None], k[:, None], v[:, None], g[:, None], b[:, None], state_in=S0[None, None])
    assert rel(O, o2[:, 0]) < 1e-12 and rel(S1, s2[0, 0]) < 1e-12


@pytest.mark.parametrize("gate", [(-0.5, 0.0), (-4.0, -1.0)])
def test_pair_inverse_is_the_block_combination_of_the_chunk_inverses(gate):
    """(I + A)^-1 over 64 rows equals [[T_a, 0], [-T_b A_ba T_a, T_b]] with T_a, T_b the two 32-row
    chunks' own inverses and A_ba the pair's A between them: the pair operator is built from the
    chunks' 32 x 32 solves."""
    d = 16
    q, k, v, g, b = _one_head(64, d, 72, gate)
    pair = oracle.chunk_operator(q, k, g, b, chunk=64)
    ta = oracle.chunk_operator(q[:32], k[:32], g[:32], b[:32])["T"]
    tb = oracle.chunk_operator(q[32:], k[32:], g[32:], b[32:])["T"]
    a_ba = pair["A"][32:, :32]
    blocks = np.block([[ta, np.zeros((32, 32))], [-tb @ a_ba @ ta, tb]])
    assert rel(blocks, pair["T"]) < 1e-12
    # a plausible slip: T_ba with the wrong sign or the factors swapped
    wrong = np.block([[ta, np.zeros((32, 32))], [-ta @ a_ba @ tb, tb]])
    assert rel(wrong, pair["T"]) > 1e-6


def test_cross_chunk_gram_gives_the_lookahead_identity():
    """[X_c; Z_c] from the exact state equals Gamma_C(c-1) [K;Q]_c S_{c-2}^T + G'_c U~_{c-1}: the
    identity that lets the state-dependent product of a chunk run one chunk early."""
    d, C = 16, 32
    q, k, v, g, b = _one_head(3 * C, d, 63)
    S = 0.05 * np.random.default_rng(64).standard_normal((d, d))
    sl = [slice(c * C, (c + 1) * C) for c in range(3)]
    op0 = oracle.chunk_operator(q[sl[0]], k[sl[0]], g[sl[0]], b[sl[0]])
    _, S_a = oracle.chunk_step(op0, q[sl[0]], k[sl[0]], v[sl[0]], S)           # S_{c-2}
    op1 = oracle.chunk_operator(q[sl[1]], k[sl[1]], g[sl[1]], b[sl[1]], k_prev=k[sl[0]])
    X1 = k[sl[1]] @ S_a.T
    U1 = op1["Tpp"] @ (v[sl[1]] - op1["Gamma"][:, None] * X1)
    Ut1 = op1["delta"][:, None] * U1                                           # U~_{c-1}
    _, S_b = oracle.chunk_step(op1, q[sl[1]], k[sl[1]], v[sl[1]], S_a)         # S_{c-1}
    op2 = oracle.chunk_operator(q[sl[2]], k[sl[2]], g[sl[2]], b[sl[2]], k_prev=k[sl[1]])
    KQ = np.concatenate([k[sl[2]], q[sl[2]]])
    direct = KQ @ S_b.T
    lookahead = op1["GammaC"] * (KQ @ S_a.T) + op2["Gp"] @ Ut1
    assert rel(lookahead, direct) < 1e-12


def test_chunk_operator_planted_mistake_is_caught():
    """A that keeps its diagonal (j <= i instead of j < i) must break the reconstruction."""
    d, L = 16, 20
    q, k, v, g, b = _one_head(L, d, 65)
    S0 = 0.05 * np.random.default_rng(66).standard_normal((d, d))
    op = oracle.chunk_operator(q, k, g, b)
    C = 32
    K = np.zeros((C, d))
    K[:L] = k
    Bt = np.zeros(C)
    Bt[:L] = b
    gam = np.cumsum(np.concatenate([g, np.zeros(C - L)]))
    D = np.exp(gam[:, None] - gam[None, :])
    i, j = np.indices((C, C))
    A_bad = np.where(j <= i, Bt[:, None] * D * (K @ K.T), 0.0)
    bad = dict(op)
    bad["Tpp"] = np.linalg.inv(np.eye(C) + A_bad) * Bt[None, :]
    O, S1 = oracle.chunk_step(bad, q, k, v, S0)
    o2, s2 = oracle.recurrence(q[:, None], k[:, None], v[:, None], g[:, None], b[:, None], state_in=S0[None, None])
    assert rel(S1, s2[0, 0]) > 1e-6


# a best-first draft tree of 8 nodes per sequence: a main chain with side branches, and a root
# sibling (parent -1); every parent precedes its child
TREE8 = [[-1, 0, 1, 1, 3, 0, -1, 6],
         [-1, 0, 0, 2, 2, 4, 1, 6]]


def _tree_inputs(B, Tk, H, d, seed):
    q, k, v, g, b, _ = rnd(B * Tk, H, d, d, seed)
    s0 = 0.05 * np.random.default_rng(seed + 1).standard_normal((B, H, d, d))
    return tuple(x.reshape((B, Tk) + x.shape[1:]) for x in (q, k, v, g, b)) + (s0,)


def test_decode_verify_tree_nodes_match_brute_force_along_their_path():
    """Every node's state and output equal the explicit-matrix expansion over the tokens on the path
    from the root to that node, starting from the committed state (left untouched)."""
    B, Tk, H, d = 2, 8, 2, 6
    q, k, v, g, b, s0 = _tree_inputs(B, Tk, H, d, 41)
    keep = s0.copy()
    o, st = oracle.decode_verify_tree(q, k, v, g, b, TREE8, s0)
    assert np.array_equal(s0, keep)
    for i in range(B):
        for t in range(Tk):
            path = oracle.tree_path(TREE8[i], t)
            assert len(path) <= 8 and path[-1] == t
            ob, sb = oracle.brute_force(q[i, path], k[i, path], v[i, path], g[i, path], b[i, path],
                                        state_in=s0[i][None])
            assert rel(st[i, t], sb[0]) < 1e-12
            assert rel(o[i, t], ob[-1]) < 1e-12


def test_decode_verify_tree_nodes_equal_the_recurrence_on_their_path():
    """Deeper random trees (up to 24 nodes): each node = the plain recurrence over its root path."""
    B, Tk, H, d = 3, 24, 2, 8
    q, k, v, g, b, s0 = _tree_inputs(B, Tk, H, d, 43)
    r = np.random.default_rng(44)
    par = np.array([[-1] + [int(r.integers(-1, t)) for t in range(1, Tk)] for _ in range(B)])
    o, st = oracle.decode_verify_tree(q, k, v, g, b, par, s0)
    for i in range(B):
        for t in range(Tk):
            path = oracle.tree_path(par[i], t)
            o2, s2 = oracle.recurrence(q[i, path], k[i, path], v[i, path], g[i, path], b[i, path],
                                       state_in=s0[i][None])
            assert rel(st[i, t], s2[0]) < 1e-13
            assert rel(o[i, t], o2[-1]) < 1e-13


def test_decode_verify_tree_special_shapes():
    """A chain tree is the linear verify; a star (every node on the committed state) is Tk
    independent single steps from that state."""
    B, Tk, H, d = 2, 5, 2, 8
    q, k, v, g, b, s0 = _tree_inputs(B, Tk, H, d, 45)
    chain = [[t - 1 for t in range(Tk)]] * B
    o1, s1 = oracle.decode_verify_tree(q, k, v, g, b, chain, s0)
    o2, s2 = oracle.decode_verify(q, k, v, g, b, s0)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    star = [[-1] * Tk] * B
    o3, s3 = oracle.decode_verify_tree(q, k, v, g, b, star, s0)
    for t in range(Tk):
        o4, s4 = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], s0)
        assert rel(o3[:, t], o4) < 1e-14 and rel(s3[:, t], s4) < 1e-14


def test_decode_verify_tree_rejects_forward_or_out_of_range_parents():
    B, Tk, H, d = 1, 4, 1, 4
    q, k, v, g, b, s0 = _tree_inputs(B, Tk, H, d, 47)
    for bad in ([[-1, 0, 2, 1]], [[-1, 0, -2, 1]], [[0, 0, 1, 2]]):
        with pytest.raises(ValueError):
            oracle.decode_verify_tree(q, k, v, g, b, bad, s0)


def test_tree_planted_mistake_is_caught():
    """A verify that ignores the tree and continues from the previous node (a chain) must fail the
    path pin on a tree that branches."""
    B, Tk, H, d = 2, 8, 2, 6
    q, k, v, g, b, s0 = _tree_inputs(B, Tk, H, d, 49)
    o_wrong, s_wrong = oracle.decode_verify(q, k, v, g, b, s0)       # the mistake: previous node
    bad = 0
    for i in range(B):
        for t in range(Tk):
            path = oracle.tree_path(TREE8[i], t)
            o2, s2 = oracle.recurrence(q[i, path], k[i, path], v[i, path], g[i, path], b[i, path],
                                       state_in=s0[i][None])
            bad += rel(s_wrong[i, t], s2[0]) > 1e-6
    assert bad > 0


# ---------------------------------------------------------------------------------------------
# planted mistakes: each variant below is one plausible error; at least one pin must reject it
# ---------------------------------------------------------------------------------------------
def _recurrence_variant(q, k, v, g, b, s0, mistake):
    T, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((T, H, dv))
    S = s0[0].copy()
    for h in range(H):
        for t in range(T):
            a = np.exp(g[t, h])
            P = np.eye(dk) - b[t, h] * np.outer(k[t, h], k[t, h])
            W = b[t, h] * np.outer(v[t, h], k[t, h])
            if mistake == "gate_on_write":
                S[h] = a * (S[h] @ P + W)
            elif mistake == "left_multiply":
                S[h] = a * (P[:dv, :dv] @ S[h]) + W if dv == dk else S[h]
            elif mistake == "sign":
                S[h] = a * S[h] @ (np.eye(dk) + b[t, h] * np.outer(k[t, h], k[t, h])) + W
            elif mistake == "no_scale":
                S[h] = a * S[h] @ P + W
            o[t, h] = S[h] @ q[t, h] / (1.0 if mistake == "no_scale" else np.sqrt(dk))
    return o, S[None]


@pytest.mark.parametrize("mistake", ["gate_on_write", "left_multiply", "sign", "no_scale"])
def test_planted_mistakes_are_caught(mistake):
    """A test-local copy of the recurrence with one planted error must disagree with the oracle on
    the pins above (hand values of case A, the beta = 1 projection)."""
    c = _parse_golden()["A"]
    q = np.array([t["q"] for t in c["tokens"]])[:, None, :]
    k = np.array([t["k"] for t in c["tokens"]])[:, None, :]
    v = np.array([t["v"] for t in c["tokens"]])[:, None, :]
    g = np.log(np.array([t["alpha"][0] for t in c["tokens"]]))[:, None]
    b = np.array([t["beta"][0] for t in c["tokens"]])[:, None]
    o, s = _recurrence_variant(q, k, v, g, b, c["S0"][None, None], mistake)
    ok_hand = np.allclose(o[:, 0] * np.sqrt(2.0), np.array(c["o"]), atol=1e-9) and np.allclose(s[0, 0], c["S"], atol=1e-9)
    # projection pin with random data
    q2, k2, v2, g2, b2, s02 = rnd(6, 1, 4, 4, 17, N=1)
    b2[:] = 1.0
    _, sv = _recurrence_variant(q2, k2, v2, g2, b2, s02, mistake)
    ok_proj = np.max(np.abs(sv[0, 0] @ k2[-1, 0] - v2[-1, 0])) < 1e-12
    assert not (ok_hand and ok_proj), "planted mistake %r passed the pins" % mistake

