"""Shared test utilities: conversions, error metrics and oracle comparisons on sampled rows."""
import numpy as np
import torch

import oracle

# Parity bars of the method: max |err| / max |ref| for outputs and final states.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def f64(t):
    """Exact widening of a (possibly bf16) tensor to a float64 numpy array."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def oracle_full(inp):
    """Full fp64 oracle of one prefill input dict (small sizes only)."""
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    s0 = None if inp["state_in"] is None else f64(inp["state_in"])
    return oracle.recurrence(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["beta"]),
                             cu_seqlens=cu, state_in=s0)


def sampled_rows_check(inp, out, state_out, picks):
    """Compare GPU outputs / final states with the oracle on sampled (sequence, head, row) triples.

    The oracle runs per head on that head's slice only, so full-size workloads stay cheap.
    Returns (max relative error of o over the sampled rows, of the final-state rows)."""
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    by_head = {}
    for (n, h, r) in picks:
        by_head.setdefault(int(h), []).append((int(n), int(r)))
    o_got, o_ref, s_got, s_ref = [], [], [], []
    for h, lst in by_head.items():
        sl = slice(h, h + 1)
        s0 = None if inp["state_in"] is None else f64(inp["state_in"][:, sl])
        samples = np.array([[n, 0, r] for (n, r) in lst], dtype=np.int64)
        orow, srow = oracle.rows(f64(inp["q"][:, sl]), f64(inp["k"][:, sl]), f64(inp["v"][:, sl]),
                                 f64(inp["g"][:, sl]), f64(inp["beta"][:, sl]), samples, cu_seqlens=cu,
                                 state_in=s0)
        og = f64(out[:, h, :])
        sg = f64(state_out[:, h]) if state_out is not None else None
        for i, (n, r) in enumerate(lst):
            a, e = cu[n], cu[n + 1]
            o_got.append(og[a:e, r])
            o_ref.append(orow[i, a:e])
            if sg is not None:
                s_got.append(sg[n, r])
                s_ref.append(srow[i])
    eo = rel_err(np.concatenate(o_got), np.concatenate(o_ref))
    es = rel_err(np.concatenate(s_got), np.concatenate(s_ref)) if s_got else 0.0
    return eo, es


def pick_rows(N, H, dv, count, seed=0, lengths=None):
    r = np.random.default_rng(seed)
    picks = set()
    while len(picks) < count:
        n = int(r.integers(N))
        if lengths is not None and lengths[n] == 0:
            continue
        picks.add((n, int(r.integers(H)), int(r.integers(dv))))
    return sorted(picks)
