"""GPU parity of gdn_chunk_prefill against the fp64 oracle (all calls go through the C ABI).

Parity bar: max |o_gpu - o_ref| / max |o_ref| <= 1e-4 for fp32 q/k/v and <= 2e-2 for bf16 q/k/v,
the same for final states relative to max |S_ref|.
"""
import numpy as np
import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import WORKLOADS, make_prefill_inputs, workload_inputs

from helpers import (OUT_TOL_BF16_ROUNDING, STATE_TOL_BF16_FP32LEVEL, TOL, f64, full_heads_check, oracle_full,
                     rel_err, sampled_rows_check)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(inp, **kw):
    return gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                 cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"], **kw)


def check_full(inp, tag=""):
    out, st = run(inp)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle_full(inp)
    eo, es = rel_err(f64(out), o_ref), rel_err(f64(st), s_ref)
    tol = TOL[inp["q"].dtype]
    print("%s o_err=%.3e s_err=%.3e tol=%g" % (tag, eo, es, tol))
    assert eo <= tol and es <= tol, (eo, es)
    return out, st


def test_tiny_fp32_workload():
    """T=128 (4 chunks), H=2, dk=dv=64, fp32, zero initial state: every output and the state."""
    check_full(workload_inputs("tiny_fp32", device=DEV), "tiny_fp32")


@pytest.mark.parametrize("T", [1, 31, 32, 33, 63, 64, 65, 200])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_ragged_lengths(T, dtype):
    inp = make_prefill_inputs([T], 3, 64, 64, dtype, "uniform", seed=T, state_std=0.05, device=DEV)
    check_full(inp, "T=%d %s" % (T, dtype))


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_head_sizes(dk, dv, dtype):
    inp = make_prefill_inputs([70, 33], 2, dk, dv, dtype, "softplus", seed=dk + dv, state_std=0.05, device=DEV)
    check_full(inp, "dk=%d dv=%d %s" % (dk, dv, dtype))


def test_varlen_with_empty_sequences():
    lengths = [0, 45, 0, 1, 96, 0]
    inp = make_prefill_inputs(lengths, 2, 64, 64, "fp32", "uniform", seed=5, state_std=0.05, device=DEV)
    out, st = check_full(inp, "varlen-empty")
    # empty sequences hand their initial state through unchanged
    for n, L in enumerate(lengths):
        if L == 0:
            assert torch.equal(st[n], inp["state_in"][n])


def test_strong_gates():
    """g down to -8 per token: per-chunk cumulative gates reach -256; local cumsums keep exp finite."""
    inp = make_prefill_inputs([160], 2, 64, 64, "fp32", "uniform", seed=7, state_std=0.05, device=DEV)
    inp["g"] = inp["g"] * 16.0
    check_full(inp, "strong-gates")


def test_strong_gates_bf16_pairs():
    """The bf16 path takes the cumulative gate over a pair of chunks (64 rows): with g down to -8 per
    token it reaches -512, so Gamma_i and Gamma_C underflow to zero in fp32 inside a pair while the
    decay ratios between nearby rows (running products) stay exact; outputs and states still match
    the oracle, states at fp32 level."""
    inp = make_prefill_inputs([200, 64, 31], 2, 128, 128, "bf16", "uniform", seed=9, state_std=0.05, device=DEV)
    inp["g"] = inp["g"] * 16.0
    out, st = check_full(inp, "strong-gates-bf16")
    o_ref, s_ref = oracle_full(inp)
    assert rel_err(f64(st), s_ref) <= STATE_TOL_BF16_FP32LEVEL


def test_null_state_in_equals_zeros():
    inp = make_prefill_inputs([100], 2, 128, 128, "bf16", "softplus", seed=8, device=DEV)
    o1, s1 = run(inp)
    inp2 = dict(inp, state_in=torch.zeros(1, 2, 128, 128, device=DEV))
    o2, s2 = run(inp2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_in_place_state():
    inp = make_prefill_inputs([77, 40], 2, 64, 128, "fp32", "uniform", seed=9, state_std=0.05, device=DEV)
    o1, s1 = run(inp)
    buf = inp["state_in"].clone()
    o2, s2 = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   cu_seqlens=inp["cu_seqlens"], state_in=buf, state_out=buf)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, buf)


def test_no_state_out():
    inp = make_prefill_inputs([50], 2, 64, 64, "fp32", "uniform", seed=10, device=DEV)
    o1, _ = run(inp)
    o2, s2 = run(inp, output_final_state=False)
    torch.cuda.synchronize()
    assert s2 is None and torch.equal(o1, o2)


def test_equal_length_without_cu_seqlens():
    inp = make_prefill_inputs([64, 64, 64], 2, 64, 64, "bf16", "softplus", seed=11, device=DEV)
    o1, s1 = run(inp)
    o2, s2 = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], num_seqs=3)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_empty_call_copies_state():
    H, d = 2, 64
    s0 = torch.randn(2, H, d, d, device=DEV)
    e = torch.empty((0, H, d), device=DEV)
    eg = torch.empty((0, H), device=DEV)
    cu = torch.zeros(3, dtype=torch.int32, device=DEV)
    out, st = gdn.gdn_chunk_prefill(e, e, e, eg, eg, cu_seqlens=cu, state_in=s0)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(st, s0) and out.numel() == 0


def test_bad_cu_seqlens_reported_on_device():
    inp = make_prefill_inputs([40, 40], 2, 64, 64, "fp32", "uniform", seed=12, device=DEV)
    out = torch.full_like(inp["v"], 7.0)
    st = torch.full((2, 2, 64, 64), 7.0, device=DEV)
    for bad in ([0, 50, 40], [0, 40, 81], [1, 40, 80]):
        cu = torch.tensor(bad, dtype=torch.int32, device=DEV)
        gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=cu, out=out,
                              state_out=st)
        assert gdn.gdn_get_device_status() == -6
        assert torch.all(out == 7.0) and torch.all(st == 7.0)
    assert gdn.gdn_get_device_status() == 0   # the word was cleared by the read


# ---------------------------------------------------------------------------------------------
# cross-call properties (Ferrite page, Design sections 06 and 07; prefix invariance)
# ---------------------------------------------------------------------------------------------
def test_split_resume_equals_one_shot():
    inp = make_prefill_inputs([300], 2, 128, 128, "fp32", "softplus", seed=13, state_std=0.05, device=DEV)
    o_full, s_full = run(inp)
    for cut in (32, 45, 128, 257):
        a = {k_: (v_[:cut] if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in inp.items()}
        a["cu_seqlens"] = torch.tensor([0, cut], dtype=torch.int32, device=DEV)
        oa, sa = run(a)
        b = {k_: (v_[cut:] if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in inp.items()}
        b["cu_seqlens"] = torch.tensor([0, 300 - cut], dtype=torch.int32, device=DEV)
        b["state_in"] = sa
        ob, sb = run(b)
        torch.cuda.synchronize()
        o_cat = torch.cat([oa, ob])
        if cut % 32 == 0:      # same chunk boundaries: bitwise equal
            assert torch.equal(o_cat, o_full) and torch.equal(sb, s_full)
        else:                  # other boundaries: equal up to rounding
            assert rel_err(f64(o_cat), f64(o_full)) < 1e-5 and rel_err(f64(sb), f64(s_full)) < 1e-5


def test_pack_equals_solo_runs_bitwise():
    lengths = [37, 64, 5, 100]
    inp = make_prefill_inputs(lengths, 2, 128, 128, "bf16", "softplus", seed=14, state_std=0.05, device=DEV)
    o, s = run(inp)
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(lengths)):
        a, e = cu[n], cu[n + 1]
        solo = {k_: (v_[a:e] if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in inp.items()}
        solo["cu_seqlens"] = torch.tensor([0, e - a], dtype=torch.int32, device=DEV)
        solo["state_in"] = inp["state_in"][n:n + 1].contiguous()
        on, sn = run(solo)
        torch.cuda.synchronize()
        assert torch.equal(on, o[a:e]) and torch.equal(sn[0], s[n])


def test_deterministic():
    inp = make_prefill_inputs([513], 4, 128, 128, "bf16", "softplus", seed=15, state_std=0.05, device=DEV)
    o1, s1 = run(inp)
    o2, s2 = run(inp)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("t", [0, 31, 32, 63, 64, 100])
def test_prefix_invariance(t):
    inp = make_prefill_inputs([160], 2, 64, 64, "fp32", "uniform", seed=16, state_std=0.05, device=DEV)
    o1, _ = run(inp)
    inp2 = dict(inp)
    gen = torch.Generator(device=DEV).manual_seed(1234)
    for name in ("q", "k", "v"):
        x = inp[name].clone()
        x[t + 1:] = torch.randn(x[t + 1:].shape, generator=gen, device=DEV)
        inp2[name] = x
    inp2["g"] = inp["g"].clone()
    inp2["g"][t + 1:] = -torch.rand(inp2["g"][t + 1:].shape, generator=gen, device=DEV)
    o2, _ = run(inp2)
    torch.cuda.synchronize()
    assert torch.equal(o1[:t + 1], o2[:t + 1])
    assert not torch.equal(o1[t + 1:], o2[t + 1:])


# ---------------------------------------------------------------------------------------------
# full-size workloads against the oracle
# ---------------------------------------------------------------------------------------------
def _bf16_fp32_level(name, eo, es):
    """The bf16 path's extra bars: final states at fp32 level, outputs within bf16 rounding."""
    print("%s fp32-level bars: s_err=%.3e (<= %g), o_err=%.3e (<= %g)"
          % (name, es, STATE_TOL_BF16_FP32LEVEL, eo, OUT_TOL_BF16_ROUNDING))
    assert es <= STATE_TOL_BF16_FP32LEVEL, (name, es)
    assert eo <= OUT_TOL_BF16_ROUNDING, (name, eo)


@pytest.mark.parametrize("name", ["prefill_4k", "varlen_resume"])
def test_full_size_workloads_every_element(name):
    """Every output element and every final-state element of the workload against the oracle (all
    heads, all rows; the oracle runs one head per host thread)."""
    inp = workload_inputs(name, device=DEV)
    out, st = run(inp)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    eo, es = full_heads_check(inp, out, st)
    tol = TOL[inp["q"].dtype]
    print("%s every element: o_err=%.3e s_err=%.3e tol=%g" % (name, eo, es, tol))
    assert eo <= tol and es <= tol
    _bf16_fp32_level(name, eo, es)


def test_long_128k_full_heads_and_sampled_rows():
    """T = 131072 (4096 sequential chunks): heads 0 and 21 in full (all 128 state rows, so every
    dv slice of the scan) and two sampled rows of each of the 32 heads."""
    name = "long_128k"
    w = WORKLOADS[name]
    inp = workload_inputs(name, device=DEV)
    out, st = run(inp)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(st).all()
    eo, es = full_heads_check(inp, out, st, heads=[0, 21])
    tol = TOL[inp["q"].dtype]
    print("%s heads 0, 21 in full: o_err=%.3e s_err=%.3e tol=%g" % (name, eo, es, tol))
    assert eo <= tol and es <= tol
    _bf16_fp32_level(name + " full heads", eo, es)
    rng = np.random.default_rng(7)
    picks = [(0, h, int(r)) for h in range(w.H) for r in rng.choice(w.dv, 2, replace=False)]
    so, ss = sampled_rows_check(inp, out, st, picks)
    print("%s 64 sampled rows over 32 heads: o_err=%.3e s_err=%.3e" % (name, so, ss))
    assert so <= tol and ss <= tol
    _bf16_fp32_level(name + " sampled rows", so, ss)
