"""GPU parity of gdn_decode_verify (multi-token speculative verify) against the fp64 oracle, and its
equivalence with chained decode steps."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import WORKLOADS, make_verify_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(d, want_states=True):
    return gdn.gdn_decode_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], want_states=want_states)


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("Tk", [1, 3, 8])
def test_verify_small(dk, dv, dtype, Tk):
    d = make_verify_inputs(5, 3, dk, dv, Tk, dtype=dtype, seed=dk + dv + Tk, device=DEV)
    keep = d["state"].clone()
    o, st = _run(d)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(d["state"], keep)            # the committed state is only read
    o_ref, s_ref = oracle.decode_verify(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                        f64(d["state"]))
    tol = TOL[d["q"].dtype]
    assert rel_err(f64(o), o_ref) <= tol
    for t in range(Tk):
        assert rel_err(f64(st[:, t]), s_ref[:, t]) <= tol


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_verify_equals_chained_decode_steps_bitwise(dtype):
    """Token t of a verify is exactly the t-th of Tk chained gdn_decode_step calls (same operations
    in the same order), for outputs and states."""
    Tk = 6
    d = make_verify_inputs(4, 5, 128, 128, Tk, dtype=dtype, seed=7, device=DEV)
    o, st = _run(d)
    S = d["state"].clone()
    for t in range(Tk):
        ot = gdn.gdn_decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                 d["g"][:, t].contiguous(), d["beta"][:, t].contiguous(), S)
        torch.cuda.synchronize()
        assert torch.equal(ot, o[:, t])
        assert torch.equal(S, st[:, t])


def test_verify_optional_outputs():
    d = make_verify_inputs(3, 2, 64, 128, 4, seed=11, device=DEV)
    o1, st1 = _run(d)
    o2, st2 = _run(d, want_states=False)
    assert st2 is None and torch.equal(o1, o2)
    # outputs not written: states alone
    st3 = torch.empty_like(st1)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = gdn.lib().gdn_decode_verify(p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]), p(d["beta"]), p(d["state"]), p(st3),
                                     None, 3, 4, 2, 64, 128, gdn.GDN_BF16,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(st1, st3)


def test_verify_rollback_to_accepted_prefix():
    """Accepting the first a drafts of each sequence = continuing from states_out[:, a-1]: a second
    verify from that state equals the tail of one verify over all tokens."""
    Tk, a = 6, 2
    d = make_verify_inputs(3, 4, 128, 128, Tk, seed=13, device=DEV)
    o, st = _run(d)
    tail = {n: d[n][:, a:].contiguous() for n in ("q", "k", "v", "g", "beta")}
    tail["state"] = st[:, a - 1].contiguous()
    o2, st2 = _run(tail)
    torch.cuda.synchronize()
    assert torch.equal(o2, o[:, a:]) and torch.equal(st2, st[:, a:])


def test_verify_full_size():
    """verify_b64_k4: B=64, H=32, dk=dv=128, 4 drafted tokens; sampled (sequence, head) states of
    every token and all outputs against the oracle."""
    w = WORKLOADS["verify_b64_k4"]
    d = make_verify_inputs(w.decode_batch, w.H, w.dk, w.dv, w.decode_steps, dtype=w.dtype, gate=w.gate, seed=w.seed,
                           state_std=w.state_std, device=DEV)
    o, st = _run(d)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    r = np.random.default_rng(5)
    bs = r.choice(w.decode_batch, 6, replace=False)
    sub = {n: f64(d[n][bs]) for n in ("q", "k", "v", "g", "beta", "state")}
    o_ref, s_ref = oracle.decode_verify(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], sub["state"])
    tol = TOL[d["q"].dtype]
    assert rel_err(f64(o[bs]), o_ref) <= tol
    assert rel_err(f64(st[bs]), s_ref) <= tol
