"""GPU parity of gdn_decode_verify_tree (drafted tokens verified as a tree) against the fp64 oracle,
and its equivalence with the linear verify (a chain tree) and with single decode steps (a star).

Cases:
- the shapes of a best-first draft tree: a main chain with side branches and root siblings;
- random trees;
- a parent index that is not -1 or an earlier token, which the device must report.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import best_first_parents, make_verify_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _random_tree(B, Tk, seed):
    r = np.random.default_rng(seed)
    return np.array([[-1] + [int(r.integers(-1, t)) for t in range(1, Tk)] for _ in range(B)], dtype=np.int32)


def _best_first(B, Tk):
    return np.array([best_first_parents(Tk)] * B, dtype=np.int32)


def _run(d, parents):
    par = torch.as_tensor(parents, dtype=torch.int32, device=DEV)
    return gdn.gdn_decode_verify_tree(d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state"])


def _check(d, parents, o, st):
    o_ref, s_ref = oracle.decode_verify_tree(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]),
                                             parents, f64(d["state"]))
    tol = TOL[d["q"].dtype]
    assert rel_err(f64(o), o_ref) <= tol
    for t in range(parents.shape[1]):
        assert rel_err(f64(st[:, t]), s_ref[:, t]) <= tol


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", ["best_first", "random"])
def test_tree_matches_oracle(dk, dv, dtype, shape):
    B, Tk = 5, 9
    d = make_verify_inputs(B, 3, dk, dv, Tk, dtype=dtype, seed=dk + 3 * dv + Tk, device=DEV)
    parents = _best_first(B, Tk) if shape == "best_first" else _random_tree(B, Tk, dk + dv)
    keep = d["state"].clone()
    o, st = _run(d, parents)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(d["state"], keep)            # the committed state is only read
    _check(d, parents, o, st)


def test_deep_random_trees_and_per_sequence_shapes():
    """Different trees for different sequences, up to 32 nodes deep."""
    B, Tk = 6, 32
    d = make_verify_inputs(B, 2, 128, 128, Tk, dtype="bf16", seed=91, device=DEV)
    parents = _random_tree(B, Tk, 92)
    parents[0] = np.arange(-1, Tk - 1)                  # one sequence is a plain chain
    o, st = _run(d, parents)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    _check(d, parents, o, st)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_chain_tree_equals_linear_verify_bitwise(dtype):
    B, Tk = 4, 6
    d = make_verify_inputs(B, 5, 128, 128, Tk, dtype=dtype, seed=93, device=DEV)
    chain = np.tile(np.arange(-1, Tk - 1, dtype=np.int32), (B, 1))
    o1, st1 = _run(d, chain)
    o2, st2 = gdn.gdn_decode_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(st1, st2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_star_tree_equals_single_decode_steps_bitwise(dtype):
    """Every node on the committed state: node t = one decode step of token t from that state."""
    B, Tk = 4, 5
    d = make_verify_inputs(B, 3, 128, 128, Tk, dtype=dtype, seed=95, device=DEV)
    star = np.full((B, Tk), -1, dtype=np.int32)
    o, st = _run(d, star)
    for t in range(Tk):
        S = d["state"].clone()
        ot = gdn.gdn_decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                 d["g"][:, t].contiguous(), d["beta"][:, t].contiguous(), S)
        torch.cuda.synchronize()
        assert torch.equal(ot, o[:, t]) and torch.equal(S, st[:, t])


def test_tree_with_library_normalisation():
    B, Tk = 3, 7
    d = make_verify_inputs(B, 2, 128, 128, Tk, dtype="bf16", seed=97, device=DEV)
    sc = torch.exp(torch.empty((B, Tk, 2, 1), device=DEV).uniform_(-2.0, 2.0))
    qr = (d["q"].float() * sc).to(torch.bfloat16)
    kr = (d["k"].float() * sc.flip(1)).to(torch.bfloat16)
    parents = _best_first(B, Tk)
    par = torch.as_tensor(parents, device=DEV)
    o, st = gdn.gdn_decode_verify_tree(qr, kr, d["v"], d["g"], d["beta"], par, d["state"], normalize_qk=True)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    qn = oracle.l2norm(f64(qr)).astype(np.float32)
    kn = oracle.l2norm(f64(kr)).astype(np.float32)
    # the library rounds the normalised vectors to bf16, as the inputs of a normalised call would be
    qn = torch.from_numpy(qn).to(torch.bfloat16).double().numpy()
    kn = torch.from_numpy(kn).to(torch.bfloat16).double().numpy()
    o_ref, s_ref = oracle.decode_verify_tree(qn, kn, f64(d["v"]), f64(d["g"]), f64(d["beta"]), parents,
                                             f64(d["state"]))
    assert rel_err(f64(o), o_ref) <= TOL[torch.bfloat16]
    assert rel_err(f64(st[:, -1]), s_ref[:, -1]) <= TOL[torch.bfloat16]


def test_bad_parent_is_reported():
    """A forward reference (parent >= t) is detected on the device; the call itself is accepted."""
    B, Tk = 2, 4
    d = make_verify_inputs(B, 2, 64, 64, Tk, dtype="bf16", seed=99, device=DEV)
    bad = np.array([[-1, 0, 3, 1], [-1, 0, 1, 2]], dtype=np.int32)
    _run(d, bad)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == -9
    assert gdn.gdn_get_device_status() == 0            # reading the status clears it
