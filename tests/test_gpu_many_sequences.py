"""Packs of more sequences than the plan kernel's 1024 threads, through the C ABI, against the oracle.

The plan kernel scans chunk counts and merges cut points in blocks of 1024 sequences. These cases
cross several blocks: 1,500 sequences of 0 to 40 tokens (many empty, most with a partial chunk);
and a pack of 1,100 sequences with cut points spread over it.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import TOL, f64, oracle_full, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_1500_short_sequences(dtype):
    r = np.random.default_rng(81)
    lengths = [int(x) for x in r.integers(0, 41, 1500)]
    lengths[0] = 0                                            # an empty first and last sequence too
    lengths[-1] = 0
    inp = make_prefill_inputs(lengths, 2, 64, 64, dtype, "softplus", seed=82, state_std=0.05, device=DEV)
    out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle_full(inp)
    tol = TOL[inp["q"].dtype]
    assert rel_err(f64(out), o_ref) <= tol and rel_err(f64(st), s_ref) <= tol


def test_1100_sequences_with_cut_points():
    r = np.random.default_rng(83)
    lengths = [int(x) for x in r.integers(0, 50, 1100)]
    inp = make_prefill_inputs(lengths, 2, 64, 64, "bf16", "softplus", seed=84, state_std=0.05, device=DEV)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    # one cut strictly inside every 7th sequence that has at least 2 tokens
    cuts = [int(starts[n] + lengths[n] // 2) for n in range(0, len(lengths), 7) if lengths[n] >= 2]
    c = torch.tensor(cuts, dtype=torch.int32, device=DEV)
    out, st, sn = gdn.gdn_chunk_prefill_cuts(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], c,
                                             cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref, sn_ref = oracle.states_at(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                            f64(inp["beta"]), cuts, cu_seqlens=inp["cu_seqlens"].cpu().numpy(),
                                            state_in=f64(inp["state_in"]))
    tol = TOL[torch.bfloat16]
    assert rel_err(f64(out), o_ref) <= tol and rel_err(f64(st), s_ref) <= tol
    assert rel_err(f64(sn), sn_ref) <= tol
