"""GPU parity of gdn_chunk_prefill_cuts (state snapshots at cut points inside a prefill) against the
fp64 oracle, and the resume property: one call with cut points and a chain of calls resumed from its
snapshots give identical results, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
SEQ = ("q", "k", "v", "g", "beta")


def run_cuts(inp, cuts):
    c = torch.tensor(cuts, dtype=torch.int32, device=DEV)
    return gdn.gdn_chunk_prefill_cuts(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], c,
                                      cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])


def run(inp):
    return gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                                 state_in=inp["state_in"])


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_cuts_against_oracle(dk, dv, dtype):
    lengths = [200, 0, 75, 130]
    inp = make_prefill_inputs(lengths, 3, dk, dv, dtype, "softplus", seed=dk + dv + 3, state_std=0.05, device=DEV)
    cuts = [1, 31, 33, 64, 100, 199, 232, 300, 321, 404]       # aligned and unaligned, several sequences
    out, st, sn = run_cuts(inp, cuts)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref, sn_ref = oracle.states_at(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                            f64(inp["beta"]), cuts, cu_seqlens=inp["cu_seqlens"].cpu().numpy(),
                                            state_in=f64(inp["state_in"]))
    tol = TOL[inp["q"].dtype]
    assert rel_err(f64(out), o_ref) <= tol
    assert rel_err(f64(st), s_ref) <= tol
    for i in range(len(cuts)):
        assert rel_err(f64(sn[i]), sn_ref[i]) <= tol, i


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_cuts_equal_resumed_calls_bitwise(dtype):
    """One call with cuts = one call per segment, each resumed from the previous snapshot."""
    T = 333
    inp = make_prefill_inputs([T], 2, 128, 128, dtype, "softplus", seed=41, state_std=0.05, device=DEV)
    cuts = [45, 96, 97, 250]
    out, st, sn = run_cuts(inp, cuts)
    bounds = [0] + cuts + [T]
    s = inp["state_in"]
    for j in range(len(bounds) - 1):
        a, b = bounds[j], bounds[j + 1]
        part = {n: inp[n][a:b] for n in SEQ}
        part["cu_seqlens"] = torch.tensor([0, b - a], dtype=torch.int32, device=DEV)
        part["state_in"] = s
        o, s = run(part)
        torch.cuda.synchronize()
        assert torch.equal(o, out[a:b]), j
        if j < len(cuts):
            assert torch.equal(s, sn[j:j + 1]), j
    assert torch.equal(s, st)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_cuts_at_chunk_boundaries_leave_the_prefill_unchanged(dtype):
    """Cuts on multiples of 32 move no chunk boundary.  fp32 path (state carried per chunk): outputs
    and final states are those of the call without cuts, bit for bit.  bf16 path (state carried per
    pair of chunks): the cut at an odd multiple of 32 (288 = 256 + 32) moves the boundaries of the
    pairs after it, so the two agree to rounding (fp32-level states, at most one bf16 step on
    outputs)."""
    inp = make_prefill_inputs([256, 96], 2, 128, 128, dtype, "softplus", seed=42, state_std=0.05, device=DEV)
    o0, s0 = run(inp)
    out, st, sn = run_cuts(inp, [64, 128, 288])
    torch.cuda.synchronize()
    if dtype == "fp32":
        assert torch.equal(out, o0) and torch.equal(st, s0)
    else:
        assert rel_err(f64(out), f64(o0)) <= 2.0 ** -7
        assert rel_err(f64(st), f64(s0)) <= 1e-5


def test_cuts_at_pair_boundaries_leave_the_bf16_prefill_unchanged():
    """Cuts on multiples of 64 from their sequence's start move no boundary of a pair of chunks, the
    unit the bf16 path carries the state by: outputs and final states are those of the call without
    cuts, bit for bit, and each snapshot is the state the recurrence reaches there."""
    inp = make_prefill_inputs([256, 200], 2, 128, 128, "bf16", "softplus", seed=44, state_std=0.05, device=DEV)
    o0, s0 = run(inp)
    cuts = [64, 192, 256 + 128]
    out, st, sn = run_cuts(inp, cuts)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(out, o0) and torch.equal(st, s0)
    _, _, ref = oracle.states_at(*(f64(inp[x]) for x in ("q", "k", "v", "g", "beta")), cuts,
                                 cu_seqlens=inp["cu_seqlens"].cpu().numpy(), state_in=f64(inp["state_in"]))
    assert rel_err(f64(sn), ref) <= 1e-5


@pytest.mark.parametrize("cuts", [[50, 40], [0], [100], [100, 100], [130, 400]])
def test_bad_cuts_are_rejected_on_the_device(cuts):
    """Not increasing, at a sequence start, at a sequence end, repeated, or past the batch: the
    device status reports it and nothing is written."""
    inp = make_prefill_inputs([100, 150], 2, 64, 64, "bf16", "softplus", seed=43, device=DEV)
    out = torch.full_like(inp["v"], float("nan"))
    c = torch.tensor(cuts, dtype=torch.int32, device=DEV)
    o, st, sn = gdn.gdn_chunk_prefill_cuts(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], c,
                                           cu_seqlens=inp["cu_seqlens"], out=out)
    assert gdn.gdn_get_device_status() == -6
    assert torch.isnan(o).all()
