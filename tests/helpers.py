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


# fp32-level bars for the bf16-input path.  Its final states are fp32 and every fp32 operand of its
# products is split into three bf16 parts (24 significant bits), so they must agree with the oracle
# to fp32 level, far inside the 2e-2 bar that the bf16 rounding of q/k/v and of the outputs needs.
# Its outputs are rounded once to bf16 (relative error <= 2^-9 of each element), so max |err| over
# max |ref| stays below 2^-8 unless the value before rounding was already off.
STATE_TOL_BF16_FP32LEVEL = 1e-5
OUT_TOL_BF16_ROUNDING = 2.0 ** -8


def _head_slices(inp, h):
    """One head's inputs as fp64 numpy arrays (exact widening) plus cu_seqlens and its state_in."""
    sl = slice(h, h + 1)
    s0 = None if inp["state_in"] is None else f64(inp["state_in"][:, sl])
    return (f64(inp["q"][:, sl]), f64(inp["k"][:, sl]), f64(inp["v"][:, sl]), f64(inp["g"][:, sl]),
            f64(inp["beta"][:, sl]), s0)


def oracle_heads(inp, heads=None, workers=None):
    """Full fp64 oracle of the chosen heads (all by default), one head per task on a thread pool: the
    C recurrence runs without the GIL, so the heads use every host core, and no process is forked.
    Returns ``{h: (o [T, dv], S [N, dv, dk])}``."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    H = inp["q"].shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    slices = {h: _head_slices(inp, h) for h in heads}

    def one(h):
        q, k, v, g, b, s0 = slices[h]
        o, s = oracle.recurrence(q, k, v, g, b, cu_seqlens=cu, state_in=s0)
        return h, o[:, 0], s[:, 0]

    with ThreadPoolExecutor(max_workers=workers or min(len(heads), os.cpu_count() or 1)) as ex:
        return {h: (o, s) for h, o, s in ex.map(one, heads)}


def full_heads_check(inp, out, state_out, heads=None):
    """max |err| / max |ref| of outputs and final states over every element of the chosen heads."""
    ref = oracle_heads(inp, heads)
    hs = sorted(ref)
    o_ref = np.stack([ref[h][0] for h in hs], axis=1)
    s_ref = np.stack([ref[h][1] for h in hs], axis=1)
    o_got = np.stack([f64(out[:, h]) for h in hs], axis=1)
    s_got = np.stack([f64(state_out[:, h]) for h in hs], axis=1)
    return rel_err(o_got, o_ref), rel_err(s_got, s_ref)

