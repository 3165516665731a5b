"""Randomised GPU parity: drawn packs of sequences, head sizes, dtypes, initial states, library
normalisation and draft trees, each checked against the fp64 oracle at the stated tolerances.

The examples are drawn by hypothesis with a fixed seed and a bounded count, so a run takes seconds
and is repeatable.
"""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, seed, settings
from hypothesis import strategies as st

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs, make_verify_inputs

from helpers import TOL, f64, oracle_full, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
SETTINGS = dict(max_examples=25, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])

lengths_st = st.lists(st.one_of(st.integers(0, 3), st.integers(30, 34), st.integers(60, 70), st.integers(0, 160)),
                      min_size=1, max_size=5)


@seed(20261202)
@settings(**SETTINGS)
@given(lengths=lengths_st, H=st.integers(1, 3), dk=st.sampled_from([64, 128]), dv=st.sampled_from([64, 128]),
       dtype=st.sampled_from(["fp32", "bf16"]), with_state=st.booleans(), normalise=st.booleans(),
       data_seed=st.integers(0, 2 ** 16))
def test_random_prefill_packs(lengths, H, dk, dv, dtype, with_state, normalise, data_seed):
    if sum(lengths) == 0:
        lengths = lengths + [1]
    inp = make_prefill_inputs(lengths, H, dk, dv, dtype, "softplus", seed=data_seed,
                              state_std=0.05 if with_state else None, device=DEV)
    q, k = inp["q"], inp["k"]
    if normalise:
        # raw vectors of random scale: the library normalises them
        sc = torch.exp(torch.empty(q.shape[:2] + (1,), device=DEV).uniform_(-2.0, 2.0))
        q, k = (q.float() * sc).to(q.dtype), (k.float() * sc.flip(0)).to(k.dtype)
    out, stt = gdn.gdn_chunk_prefill(q, k, inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                                     state_in=inp["state_in"], normalize_qk=normalise)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    ref_in = dict(inp)
    if normalise:
        # the library rounds the normalised vectors to the storage dtype; so does the reference
        ref_in["q"] = torch.from_numpy(oracle.l2norm(f64(q)).astype(np.float32)).to(q.dtype)
        ref_in["k"] = torch.from_numpy(oracle.l2norm(f64(k)).astype(np.float32)).to(k.dtype)
    o_ref, s_ref = oracle_full(ref_in)
    tol = TOL[inp["q"].dtype]
    assert rel_err(f64(out), o_ref) <= tol and rel_err(f64(stt), s_ref) <= tol


@seed(20261203)
@settings(**SETTINGS)
@given(B=st.integers(1, 4), Tk=st.integers(1, 12), dk=st.sampled_from([64, 128]), dv=st.sampled_from([64, 128]),
       dtype=st.sampled_from(["fp32", "bf16"]), data=st.data())
def test_random_verify_trees(B, Tk, dk, dv, dtype, data):
    parents = np.array([[data.draw(st.integers(-1, t - 1)) for t in range(Tk)] for _ in range(B)], dtype=np.int32)
    d = make_verify_inputs(B, 2, dk, dv, Tk, dtype=dtype, seed=7 * int(np.abs(parents).sum()) + Tk, device=DEV)
    o, s = gdn.gdn_decode_verify_tree(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                      torch.as_tensor(parents, device=DEV), d["state"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle.decode_verify_tree(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                             parents, f64(d["state"]))
    tol = TOL[d["q"].dtype]
    assert rel_err(f64(o), o_ref) <= tol and rel_err(f64(s), s_ref) <= tol
