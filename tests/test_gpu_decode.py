"""GPU parity of gdn_decode_step against the fp64 oracle, and decode/prefill consistency."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import WORKLOADS, make_decode_inputs, make_prefill_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_step_small(dk, dv, dtype):
    d = make_decode_inputs(5, 3, dk, dv, steps=4, dtype=dtype, seed=dk + dv, device=DEV)
    S = d["state"].clone()
    ref_s = f64(d["state"])
    for s in range(4):
        o = gdn.gdn_decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s], S)
        torch.cuda.synchronize()
        o_ref, ref_s = oracle.decode_step(f64(d["q"][s]), f64(d["k"][s]), f64(d["v"][s]), f64(d["g"][s]),
                                          f64(d["beta"][s]), ref_s)
        tol = TOL[d["q"].dtype]
        assert rel_err(f64(o), o_ref) <= tol
        assert rel_err(f64(S), ref_s) <= tol


def test_decode_without_output():
    d = make_decode_inputs(2, 2, 128, 128, steps=1, device=DEV)
    S1, S2 = d["state"].clone(), d["state"].clone()
    gdn.gdn_decode_step(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], S1)
    lib = gdn.lib()
    import ctypes
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.gdn_decode_step(p(d["q"][0]), p(d["k"][0]), p(d["v"][0]), p(d["g"][0]), p(d["beta"][0]), p(S2),
                             None, 2, 2, 128, 128, 1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(S1, S2)


def test_decode_chain_full_size():
    """B=64, H=32, dk=dv=128, 1000 chained steps with fresh inputs each step; the state after the
    chain is checked against the oracle on sampled (sequence, head) states (all rows)."""
    w = WORKLOADS["decode_b64"]
    d = make_decode_inputs(w.decode_batch, w.H, w.dk, w.dv, w.decode_steps, dtype=w.dtype, gate=w.gate,
                           seed=w.seed, state_std=w.state_std, device=DEV)
    S = d["state"].clone()
    outs = []
    for s in range(w.decode_steps):
        o = gdn.gdn_decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s], S)
        if s == w.decode_steps - 1:
            outs.append(o)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    r = np.random.default_rng(3)
    errs_s, errs_o = [], []
    got_s, ref_s, got_o, ref_o = [], [], [], []
    for _ in range(6):
        b, h = int(r.integers(w.decode_batch)), int(r.integers(w.H))
        q = f64(d["q"][:, b, h])[:, None, :]
        k = f64(d["k"][:, b, h])[:, None, :]
        v = f64(d["v"][:, b, h])[:, None, :]
        g = f64(d["g"][:, b, h])[:, None]
        be = f64(d["beta"][:, b, h])[:, None]
        o_ref, s_ref = oracle.recurrence(q, k, v, g, be, state_in=f64(d["state"][b, h])[None, None])
        got_s.append(f64(S[b, h]))
        ref_s.append(s_ref[0, 0])
        got_o.append(f64(outs[0][b, h]))
        ref_o.append(o_ref[-1, 0])
    es = rel_err(np.array(got_s), np.array(ref_s))
    eo = rel_err(np.array(got_o), np.array(ref_o))
    print("decode chain: state err %.3e, last-output err %.3e" % (es, eo))
    assert es <= TOL[torch.bfloat16] and eo <= TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_steps_equal_prefill(dtype):
    """T decode steps from S_0 give the same outputs and state as one prefill of the T tokens."""
    T, H, d = 40, 2, 128
    inp = make_prefill_inputs([T], H, d, d, dtype, "uniform", seed=21, state_std=0.05, device=DEV)
    out_p, st_p = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                        cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    S = inp["state_in"].clone()
    outs = []
    for t in range(T):
        outs.append(gdn.gdn_decode_step(inp["q"][t:t + 1], inp["k"][t:t + 1], inp["v"][t:t + 1],
                                        inp["g"][t:t + 1], inp["beta"][t:t + 1], S))
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == "fp32" else 1e-2
    assert rel_err(f64(torch.cat(outs)), f64(out_p)) <= tol
    assert rel_err(f64(S), f64(st_p)) <= 1e-5
