"""GPU parity with GDN_QK_L2NORM: q and k passed raw (vectors of widely different lengths) and
normalised by the library, against the fp64 oracle run on l2-normalised inputs."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_decode_inputs, make_prefill_inputs, make_verify_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def unnormalise(x, seed):
    """Scale every (token, head) vector by a factor in [0.05, 20]: raw, un-normalised inputs."""
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    s = torch.exp(torch.empty(x.shape[:-1] + (1,), device=DEV).uniform_(np.log(0.05), np.log(20.0), generator=gen))
    return (x.float() * s).to(x.dtype)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_prefill_normalises_raw_qk(dk, dv, dtype):
    inp = make_prefill_inputs([150, 33, 0, 90], 3, dk, dv, dtype, "softplus", seed=dk + dv + 61, state_std=0.05,
                              device=DEV)
    q, k = unnormalise(inp["q"], 1), unnormalise(inp["k"], 2)
    out, st = gdn.gdn_chunk_prefill(q, k, inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                                    state_in=inp["state_in"], normalize_qk=True)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle.recurrence(oracle.l2norm(f64(q)), oracle.l2norm(f64(k)), f64(inp["v"]), f64(inp["g"]),
                                     f64(inp["beta"]), cu_seqlens=inp["cu_seqlens"].cpu().numpy(),
                                     state_in=f64(inp["state_in"]))
    tol = TOL[q.dtype]
    assert rel_err(f64(out), o_ref) <= tol and rel_err(f64(st), s_ref) <= tol


def test_prefill_cuts_normalises_raw_qk():
    inp = make_prefill_inputs([300], 2, 128, 128, "bf16", "softplus", seed=62, state_std=0.05, device=DEV)
    q, k = unnormalise(inp["q"], 3), unnormalise(inp["k"], 4)
    cuts = [70, 190]
    c = torch.tensor(cuts, dtype=torch.int32, device=DEV)
    out, st, sn = gdn.gdn_chunk_prefill_cuts(q, k, inp["v"], inp["g"], inp["beta"], c, cu_seqlens=inp["cu_seqlens"],
                                             state_in=inp["state_in"], normalize_qk=True)
    torch.cuda.synchronize()
    o_ref, s_ref, sn_ref = oracle.states_at(oracle.l2norm(f64(q)), oracle.l2norm(f64(k)), f64(inp["v"]), f64(inp["g"]),
                                            f64(inp["beta"]), cuts, cu_seqlens=inp["cu_seqlens"].cpu().numpy(),
                                            state_in=f64(inp["state_in"]))
    tol = TOL[q.dtype]
    assert rel_err(f64(out), o_ref) <= tol and rel_err(f64(st), s_ref) <= tol
    assert rel_err(f64(sn), sn_ref) <= tol


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_and_verify_normalise_raw_qk(dk, dv, dtype):
    d = make_decode_inputs(4, 3, dk, dv, steps=1, dtype=dtype, seed=63 + dk, device=DEV)
    q, k = unnormalise(d["q"][0], 5), unnormalise(d["k"][0], 6)
    S = d["state"].clone()
    o = gdn.gdn_decode_step(q, k, d["v"][0], d["g"][0], d["beta"][0], S, normalize_qk=True)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode_step(oracle.l2norm(f64(q)), oracle.l2norm(f64(k)), f64(d["v"][0]), f64(d["g"][0]),
                                      f64(d["beta"][0]), f64(d["state"]))
    tol = TOL[q.dtype]
    assert rel_err(f64(o), o_ref) <= tol and rel_err(f64(S), s_ref) <= tol

    w = make_verify_inputs(4, 3, dk, dv, 3, dtype=dtype, seed=64 + dk, device=DEV)
    qv, kv = unnormalise(w["q"], 7), unnormalise(w["k"], 8)
    ov, sv = gdn.gdn_decode_verify(qv, kv, w["v"], w["g"], w["beta"], w["state"], normalize_qk=True)
    torch.cuda.synchronize()
    ov_ref, sv_ref = oracle.decode_verify(oracle.l2norm(f64(qv)), oracle.l2norm(f64(kv)), f64(w["v"]), f64(w["g"]),
                                          f64(w["beta"]), f64(w["state"]))
    assert rel_err(f64(ov), ov_ref) <= tol and rel_err(f64(sv), sv_ref) <= tol


def test_decode_steps_equal_prefill_with_raw_qk():
    """The prefill's pre-pass and the decode kernel normalise the same way: T decode steps from a
    state equal one prefill over the same T tokens to rounding."""
    T = 40
    inp = make_prefill_inputs([T], 2, 128, 128, "fp32", "softplus", seed=65, state_std=0.05, device=DEV)
    q, k = unnormalise(inp["q"], 9), unnormalise(inp["k"], 10)
    out, st = gdn.gdn_chunk_prefill(q, k, inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                                    state_in=inp["state_in"], normalize_qk=True)
    S = inp["state_in"].clone()
    outs = []
    for t in range(T):
        outs.append(gdn.gdn_decode_step(q[t:t + 1], k[t:t + 1], inp["v"][t:t + 1], inp["g"][t:t + 1],
                                        inp["beta"][t:t + 1], S, normalize_qk=True))
    torch.cuda.synchronize()
    assert rel_err(f64(torch.cat(outs)), f64(out)) < 1e-5 and rel_err(f64(S), f64(st)) < 1e-5
