"""The seeded synthetic inputs (linear_attention_10_b200/workloads.py) follow their stated recipe.

Both sides of every parity test draw from these generators, so a drift in them would change every
workload without failing a parity check. The recipe: one generator per call, drawn in the order q, k,
v, g, beta, state; q and k standard normal, L2-normalised per (token, head) in fp32, then stored in the
storage dtype; v standard normal; beta = sigmoid(N(0, 1)); g = -0.1 softplus(N(0, 1)) or uniform on
[-0.5, 0); initial states N(0, 0.05^2). The named workloads fix their shapes: H = 32 heads of
d = 128 for a 4K prompt, a packed resume of four sequences and a 128K prompt; a small fp32 case.
"""
import torch

from linear_attention_10_b200.workloads import (WORKLOADS, cu_seqlens_of, make_decode_inputs,
                                                make_prefill_inputs, make_verify_inputs)


def test_named_workload_shapes():
    w = WORKLOADS
    assert (w["prefill_4k"].lengths, w["prefill_4k"].H, w["prefill_4k"].dk, w["prefill_4k"].dv) == ([4096], 32, 128, 128)
    assert w["prefill_4k"].dtype == "bf16" and w["prefill_4k"].gate == "softplus"
    assert w["varlen_resume"].lengths == [8192, 3000, 517, 13000] and w["varlen_resume"].state_std == 0.05
    # ragged tails against the chunk of 32: 0, 24, 5, 8 rows
    assert [L % 32 for L in w["varlen_resume"].lengths] == [0, 24, 5, 8]
    assert w["long_128k"].lengths == [131072] and w["long_128k"].H == 32
    t = w["tiny_fp32"]
    assert (t.lengths, t.H, t.dk, t.dv, t.dtype, t.gate) == ([128], 2, 64, 64, "fp32", "uniform")


def test_prefill_inputs_follow_the_recipe():
    lens = [300, 0, 1000, 17]
    inp = make_prefill_inputs(lens, H=4, dk=64, dv=32, dtype="bf16", gate="softplus", seed=3, state_std=0.05)
    T = sum(lens)
    assert inp["q"].shape == (T, 4, 64) and inp["k"].shape == (T, 4, 64) and inp["v"].shape == (T, 4, 32)
    assert inp["q"].dtype == torch.bfloat16 and inp["g"].dtype == torch.float32
    assert inp["cu_seqlens"].tolist() == [0, 300, 300, 1300, 1317]
    assert inp["state_in"].shape == (4, 4, 32, 64)
    # unit rows up to the bf16 rounding of each element
    for x in ("q", "k"):
        n = inp[x].float().norm(dim=-1)
        assert torch.all((n - 1).abs() < 1e-2)
    assert torch.all((inp["beta"] > 0) & (inp["beta"] < 1))
    g = inp["g"]
    assert torch.all(g < 0)
    # -0.1 softplus(z): the median is -0.1 ln 2
    assert abs(float(g.median()) + 0.1 * 0.6931) < 0.005
    assert abs(float(inp["state_in"].std()) - 0.05) < 0.002
    assert abs(float(inp["v"].float().std()) - 1.0) < 0.02


def test_uniform_gate_range():
    inp = make_prefill_inputs([4000], H=2, dk=64, dv=64, dtype="fp32", gate="uniform", seed=5)
    g = inp["g"]
    assert float(g.min()) >= -0.5 and float(g.max()) < 0
    assert abs(float(g.mean()) + 0.25) < 0.01
    assert inp["state_in"] is None and inp["q"].dtype == torch.float32


def test_inputs_are_reproducible_from_the_seed():
    a = make_prefill_inputs([200, 33], H=2, dk=64, dv=64, seed=11, state_std=0.05)
    b = make_prefill_inputs([200, 33], H=2, dk=64, dv=64, seed=11, state_std=0.05)
    c = make_prefill_inputs([200, 33], H=2, dk=64, dv=64, seed=12, state_std=0.05)
    for n in ("q", "k", "v", "g", "beta", "state_in"):
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])


def test_verify_inputs_are_a_decode_chain_in_token_order():
    d = make_decode_inputs(3, 2, 64, 64, 4, seed=7)
    v = make_verify_inputs(3, 2, 64, 64, 4, seed=7)
    assert torch.equal(v["state"], d["state"])
    for n in ("q", "k", "v", "g", "beta"):
        assert torch.equal(v[n], d[n].transpose(0, 1))


def test_cu_seqlens_of():
    assert cu_seqlens_of([]).tolist() == [0]
    assert cu_seqlens_of([5, 0, 7]).tolist() == [0, 5, 5, 12]
    assert cu_seqlens_of([5]).dtype == torch.int32
