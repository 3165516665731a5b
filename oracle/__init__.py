"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The product path (``linear_attention_10_b200``) never imports, links or runs it, and this
package imports nothing from the product path: the two share no code.

What is computed and why (each function cites its source):

* ``recurrence``  -- the gated delta rule token by token (``gdn_oracle.c``), the definition.
* ``rows``        -- the same recurrence restricted to chosen rows of the state, for sampled checks
                     of full-size workloads.
* ``chunked``     -- the chunkwise WY/UT evaluation of the recurrence in fp64 for any chunk size
                     (Ferrite project page, Design section 03 "Chunked Gated DeltaNet": chunks of
                     32 rows, WY/UT form).
* ``brute_force`` -- explicit d x d matrix products of the unrolled recurrence, numpy, for T <= 8.
* ``decode_step``, ``decode_verify``, ``decode_verify_tree`` -- the recurrence one token at a time
                     from a given state: one step, a chain of drafted tokens, and a tree of drafted
                     tokens where each node continues from its parent's state (Ferrite project page,
                     Design section 04: drafts checked in one pass as a best-first tree); ``tree_path`` lists the
                     nodes from the root to a node.
* ``states_at``   -- the recurrence with the state captured at cut points (Design section 07).
* ``chunk_operator``, ``chunk_step`` -- one chunk's state-independent WY/UT quantities (the decay
                     matrix, A, T = (I + A)^-1, T'' = T diag(beta), P, P T'', the cross-chunk Gram G'
                     and the gates) and the chunk step built from them, for checks of one stage.
* ``l2norm``      -- the L2 normalisation the method's q and k carry.

The recurrence (published gated delta rule, Yang, Kautz and Hatamizadeh, "Gated Delta Networks"):
``S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T``, ``o_t = S_t q_t / sqrt(dk)``.
Layouts: q, k ``[T, H, dk]``; v, o ``[T, H, dv]``; g, beta ``[T, H]``; state ``[N, H, dv, dk]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``libgdn_oracle.so`` with gcc (fp64, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.gdn_oracle_recurrence.argtypes = [dp, dp, dp, dp, dp, lp, i64, dp, dp, dp, i64, i64, i64]
        lib.gdn_oracle_rows.argtypes = [dp, dp, dp, dp, dp, lp, i64, dp, i64, i64, i64, i64,
                                        lp, lp, lp, dp, dp]
        lib.gdn_oracle_chunked.argtypes = [dp, dp, dp, dp, dp, lp, i64, dp, dp, dp, i64, i64, i64, i64]
        for f in (lib.gdn_oracle_recurrence, lib.gdn_oracle_rows, lib.gdn_oracle_chunked):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _d(a):
    """Contiguous fp64 copy (widening is exact for bf16 / fp32 inputs)."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, typ=ctypes.c_double):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(typ))


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        return np.array([0, T], dtype=np.int64)
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def _prep(q, k, v, g, beta, cu_seqlens, state_in):
    q, k, v, g, beta = (_d(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = _cu(cu_seqlens, T)
    assert k.shape == (T, H, dk) and v.shape[:2] == (T, H) and g.shape == (T, H) == beta.shape
    assert cu[-1] == T
    N = len(cu) - 1
    s0 = None
    if state_in is not None:
        s0 = _d(state_in)
        assert s0.shape == (N, H, dv, dk)
    return q, k, v, g, beta, cu, s0, T, H, dk, dv, N


def recurrence(q, k, v, g, beta, cu_seqlens=None, state_in=None):
    """Token-by-token gated delta rule in fp64.  Returns ``(o [T,H,dv], state [N,H,dv,dk])``."""
    q, k, v, g, beta, cu, s0, T, H, dk, dv, N = _prep(q, k, v, g, beta, cu_seqlens, state_in)
    out = np.zeros((T, H, dv))
    st = np.zeros((N, H, dv, dk))
    rc = _load().gdn_oracle_recurrence(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                       _ptr(cu, ctypes.c_int64), N, _ptr(s0), _ptr(out), _ptr(st),
                                       H, dk, dv)
    if rc != 0:
        raise ValueError("gdn_oracle_recurrence failed: %d" % rc)
    return out, st


def rows(q, k, v, g, beta, samples, cu_seqlens=None, state_in=None):
    """Recurrence for sampled state rows.

    ``samples`` is an int array ``[n, 3]`` of (sequence, head, row).  Returns ``(o_rows, s_rows)``:
    ``o_rows[i, t]`` = o_t[h, r] for t in that sequence (NaN elsewhere), ``s_rows[i]`` = final
    state row ``S[n, h, r, :]``.
    """
    q, k, v, g, beta, cu, s0, T, H, dk, dv, N = _prep(q, k, v, g, beta, cu_seqlens, state_in)
    smp = np.ascontiguousarray(np.asarray(samples, dtype=np.int64).reshape(-1, 3))
    n = smp.shape[0]
    si, hi, ri = (np.ascontiguousarray(smp[:, j]) for j in range(3))
    o_rows = np.full((n, T), np.nan)
    s_rows = np.zeros((n, dk))
    rc = _load().gdn_oracle_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(cu, ctypes.c_int64), N, _ptr(s0), H, dk, dv, n,
                                 _ptr(si, ctypes.c_int64), _ptr(hi, ctypes.c_int64),
                                 _ptr(ri, ctypes.c_int64), _ptr(o_rows), _ptr(s_rows))
    if rc != 0:
        raise ValueError("gdn_oracle_rows failed: %d" % rc)
    return o_rows, s_rows


def chunked(q, k, v, g, beta, chunk, cu_seqlens=None, state_in=None):
    """Chunkwise WY/UT evaluation in fp64 with chunk size ``chunk``.  Same returns as ``recurrence``."""
    q, k, v, g, beta, cu, s0, T, H, dk, dv, N = _prep(q, k, v, g, beta, cu_seqlens, state_in)
    out = np.zeros((T, H, dv))
    st = np.zeros((N, H, dv, dk))
    rc = _load().gdn_oracle_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(cu, ctypes.c_int64), N, _ptr(s0), _ptr(out), _ptr(st),
                                    H, dk, dv, int(chunk))
    if rc != 0:
        raise ValueError("gdn_oracle_chunked failed: %d" % rc)
    return out, st


def decode_step(q, k, v, g, beta, state):
    """One recurrent step for B independent sequences: inputs ``[B, H, d]`` / ``[B, H]``, state
    ``[B, H, dv, dk]``.  This is the recurrence over B sequences of length one."""
    B = np.asarray(q).shape[0]
    return recurrence(q, k, v, g, beta, cu_seqlens=np.arange(B + 1), state_in=state)


def l2norm(x, eps=1e-12):
    """L2 normalisation of every vector along the last axis in fp64, x / max(||x||_2, eps): the
    step that makes q_t and k_t the unit vectors the recurrence is defined on (inputs of the
    method are L2-normalised per token and head)."""
    x = _d(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def states_at(q, k, v, g, beta, cuts, cu_seqlens=None, state_in=None):
    """The recurrence with the state captured at token offsets ``cuts`` (each strictly inside a
    sequence; Ferrite project page, Design section 07, turn-boundary snapshots).  Each sequence is
    run segment by segment between its cuts, carrying the state.  Returns ``(o, state,
    snapshots [len(cuts), H, dv, dk])``."""
    q, k, v, g, beta = (_d(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    cuts = [int(c) for c in np.asarray(cuts).reshape(-1)]
    out = np.zeros((T, H, dv))
    st = np.zeros((N, H, dv, dk))
    snaps = np.zeros((len(cuts), H, dv, dk))
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        inner = [(i, c) for i, c in enumerate(cuts) if a < c < b]
        s = np.zeros((1, H, dv, dk)) if state_in is None else _d(state_in)[n:n + 1].copy()
        bounds = [a] + [c for _, c in inner] + [b]
        for j in range(len(bounds) - 1):
            lo, hi = bounds[j], bounds[j + 1]
            o, s = recurrence(q[lo:hi], k[lo:hi], v[lo:hi], g[lo:hi], beta[lo:hi], state_in=s)
            out[lo:hi] = o
            if j < len(inner):
                snaps[inner[j][0]] = s[0]
        st[n] = s[0]
    return out, st, snaps


def chunk_operator(q, k, g, beta, k_prev=None, chunk=32):
    """The state-independent quantities of one chunk of one head in the chunkwise WY/UT form (Ferrite
    project page, Design section 03: chunks of 32 rows, WY/UT form), in fp64.  Inputs: q, k
    ``[L, dk]``, g, beta ``[L]`` with L <= chunk rows (the rest of the chunk is padding: g = 0,
    beta = 0, q = k = 0), k_prev ``[chunk, dk]`` the previous chunk's keys or None.  With gamma_i the
    chunk-local cumulative sum of g and D_ij = exp(gamma_i - gamma_j):

      A = strictly-lower(diag(beta) (D o K K^T)),  T = (I + A)^-1,  T'' = T diag(beta),
      P = lower-incl-diagonal(D o Q K^T),          G' = [K; Q] K_prev^T,
      Gamma_i = exp(gamma_i),  delta_i = exp(gamma_C - gamma_i),  Gamma_C = exp(gamma_C).

    Returns a dict of numpy arrays: A, T, Tpp (T''), P, PTpp (P T''), Gp (G', zeros without k_prev),
    Gamma, delta, GammaC."""
    q, k = _d(q), _d(k)
    g, beta = _d(g).reshape(-1), _d(beta).reshape(-1)
    L, dk = k.shape
    if L > chunk:
        raise ValueError("at most %d rows" % chunk)
    Q = np.zeros((chunk, dk))
    K = np.zeros((chunk, dk))
    G = np.zeros(chunk)
    Bt = np.zeros(chunk)
    Q[:L], K[:L], G[:L], Bt[:L] = q, k, g, beta
    gam = np.cumsum(G)
    D = np.exp(gam[:, None] - gam[None, :])
    i, j = np.indices((chunk, chunk))
    A = np.where(j < i, Bt[:, None] * D * (K @ K.T), 0.0)
    T = np.linalg.inv(np.eye(chunk) + A)
    Tpp = T * Bt[None, :]
    P = np.where(j <= i, D * (Q @ K.T), 0.0)
    KQ = np.concatenate([K, Q], axis=0)
    Gp = np.zeros((2 * chunk, chunk)) if k_prev is None else KQ @ _d(k_prev).T
    return dict(A=A, T=T, Tpp=Tpp, P=P, PTpp=P @ Tpp, Gp=Gp, Gamma=np.exp(gam), delta=np.exp(gam[-1] - gam),
                GammaC=float(np.exp(gam[-1])))


def chunk_step(op, q, k, v, state, chunk=32):
    """One chunk of one head from the quantities of ``chunk_operator``: with X = K S0^T, Z = Q S0^T,
    U = T'' (V - diag(Gamma) X), the outputs O = s (diag(Gamma) Z + P U) and the state after the
    chunk S1 = Gamma_C S0 + (diag(delta) U)^T K.  Inputs q, k ``[L, dk]``, v ``[L, dv]``, state
    ``[dv, dk]``; returns (O ``[L, dv]``, S1)."""
    q, k, v, S0 = _d(q), _d(k), _d(v), _d(state)
    L, dk = k.shape
    dv = v.shape[1]
    Q = np.zeros((chunk, dk))
    K = np.zeros((chunk, dk))
    V = np.zeros((chunk, dv))
    Q[:L], K[:L], V[:L] = q, k, v
    X, Z = K @ S0.T, Q @ S0.T
    U = op["Tpp"] @ (V - op["Gamma"][:, None] * X)
    O = (op["Gamma"][:, None] * Z + op["P"] @ U) / np.sqrt(dk)
    S1 = op["GammaC"] * S0 + (op["delta"][:, None] * U).T @ K
    return O[:L], S1


def decode_verify(q, k, v, g, beta, state):
    """Tk speculative tokens per sequence run in order from ``state`` (which is not modified):
    inputs ``[B, Tk, H, d]`` / ``[B, Tk, H]``.  Returns ``(out [B, Tk, H, dv], states [B, Tk, H, dv,
    dk])`` with the state after each token -- the decode step applied Tk times."""
    q, k, v, g, beta = (_d(x) for x in (q, k, v, g, beta))
    B, Tk, H, dk = q.shape
    dv = v.shape[3]
    out = np.zeros((B, Tk, H, dv))
    states = np.zeros((B, Tk, H, dv, dk))
    S = _d(state).copy()
    for t in range(Tk):
        o, S = decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        out[:, t] = o
        states[:, t] = S
    return out, states


def decode_verify_tree(q, k, v, g, beta, parents, state):
    """Tk drafted tokens per sequence arranged as a tree (Ferrite project page, Design section 04:
    the big model checks the drafts in a single pass, arranged as a tree grown best-first).  Node t of sequence b follows
    node ``parents[b, t]`` (an earlier node, < t) or, when that is -1, the committed ``state`` (not
    modified): its state is the decode step of its token applied to its parent's state.  Inputs as
    ``decode_verify`` plus ``parents`` int ``[B, Tk]``.  Returns ``(out [B, Tk, H, dv], states
    [B, Tk, H, dv, dk])``; a chain (parents[b, t] = t - 1) gives exactly ``decode_verify``."""
    q, k, v, g, beta = (_d(x) for x in (q, k, v, g, beta))
    par = np.asarray(parents, dtype=np.int64)
    B, Tk, H, dk = q.shape
    dv = v.shape[3]
    if par.shape != (B, Tk):
        raise ValueError("parents must be [B, Tk]")
    s0 = _d(state)
    out = np.zeros((B, Tk, H, dv))
    states = np.zeros((B, Tk, H, dv, dk))
    for b in range(B):
        for t in range(Tk):
            p = int(par[b, t])
            if not -1 <= p < t:
                raise ValueError("node %d of sequence %d has parent %d: it must be -1 or an earlier node" % (t, b, p))
            before = s0[b:b + 1] if p < 0 else states[b:b + 1, p]
            o, S = decode_step(q[b:b + 1, t], k[b:b + 1, t], v[b:b + 1, t], g[b:b + 1, t], beta[b:b + 1, t], before)
            out[b, t] = o[0]
            states[b, t] = S[0]
    return out, states


def tree_path(parents_row, t):
    """The nodes from the root down to node t (inclusive) of one sequence's tree, in order."""
    path = []
    while t >= 0:
        path.append(int(t))
        t = int(parents_row[t])
    return path[::-1]


def brute_force(q, k, v, g, beta, state_in=None):
    """Unrolled recurrence with explicit matrices, one sequence, T <= 8 (numpy, fp64).

    With A_t = exp(g_t) (I - beta_t k_t k_t^T) and B_t = beta_t v_t k_t^T:
    ``S_t = S_0 A_1 ... A_t + sum_{j<=t} B_j A_{j+1} ... A_t``.  Each partial product is formed
    explicitly as a d x d matrix; nothing is shared with the loop in ``gdn_oracle.c``.
    """
    q, k, v, g, beta = (_d(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    assert T <= 8, "brute force is for tiny cases only"
    out = np.zeros((T, H, dv))
    st = np.zeros((H, dv, dk))
    eye = np.eye(dk)
    for h in range(H):
        S0 = np.zeros((dv, dk)) if state_in is None else _d(state_in)[0, h]
        A = [np.exp(g[t, h]) * (eye - beta[t, h] * np.outer(k[t, h], k[t, h])) for t in range(T)]
        Bm = [beta[t, h] * np.outer(v[t, h], k[t, h]) for t in range(T)]
        for t in range(T):
            prod = eye.copy()
            for s in range(t + 1):
                prod = prod @ A[s]
            St = S0 @ prod
            for j in range(t + 1):
                tail = eye.copy()
                for s in range(j + 1, t + 1):
                    tail = tail @ A[s]
                St = St + Bm[j] @ tail
            out[t, h] = St @ q[t, h] / np.sqrt(dk)
            if t == T - 1:
                st[h] = St
    return out, st[None]
