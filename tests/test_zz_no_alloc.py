"""The allocation-free prefill entry point, called through the C ABI.

gdn_chunk_prefill_noalloc serves callers that cannot allocate device memory at the moment they run a
prefill: an inference engine that plans all of its GPU memory at start-up and forbids cudaMalloc
afterwards, or code on a latency-critical path where cudaMalloc/cudaFree could block or synchronise
the device.  Instead of a caller workspace it uses a fixed scratch array inside the library.

These checks run it through the C ABI and compare it with gdn_chunk_prefill (caller workspace): the
two run the same kernels on the same inputs, so their results must be the same bits.  Two calls in a
row make the second one run on scratch that still holds the first call's contents.  One case is
also held against the fp64 oracle, and the size limit is checked at its edge: the largest problem
whose workspace fits the scratch runs, one token more is refused, and the GDN_QK_L2NORM flag (whose
normalised q/k copies also live in the scratch) lowers the limit.  This file is collected last on
purpose.
"""
import ctypes

import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import STATE_TOL_BF16_FP32LEVEL, TOL, f64, oracle_full, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH_BYTES = 64 << 20
GDN_ERR_WORKSPACE = -5


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _code(q, norm=False):
    return (gdn.GDN_BF16 if q.dtype == torch.bfloat16 else gdn.GDN_F32) | (gdn.GDN_QK_L2NORM if norm else 0)


def _noalloc(inp, out, state_out, norm=False):
    q = inp["q"]
    T, H, dk = q.shape
    dv = inp["v"].shape[2]
    N = inp["cu_seqlens"].numel() - 1
    return gdn.lib().gdn_chunk_prefill_noalloc(
        _p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["g"]), _p(inp["beta"]), _p(inp["cu_seqlens"]), N, T,
        _p(inp["state_in"]), _p(out), _p(state_out), H, dk, dv, _code(q, norm),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _run_both(inp, norm=False):
    """(workspace entry point's out, state), (no-alloc entry point's out, state, return code)."""
    ref_o, ref_s = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                         cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"],
                                         normalize_qk=norm)
    out = torch.full_like(ref_o, float("nan"))
    st = torch.full_like(ref_s, float("nan"))
    rc = _noalloc(inp, out, st, norm)
    torch.cuda.synchronize()
    return (ref_o, ref_s), (out, st, rc)


def _largest_fitting_tokens(H, dk, dv, code, N=1):
    """Largest total token count whose workspace (gdn_chunk_prefill_workspace_bytes_ex) fits the
    scratch, by bisection on the library's own size function."""
    lo, hi = 0, 1 << 22
    assert gdn.workspace_bytes(lo, N, H, dk, dv, code) <= SCRATCH_BYTES
    assert gdn.workspace_bytes(hi, N, H, dk, dv, code) > SCRATCH_BYTES
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if gdn.workspace_bytes(mid, N, H, dk, dv, code) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_equals_workspace_entry_point_twice(dtype):
    cases = [
        make_prefill_inputs([1000, 77, 2500], 8, 128, 128, dtype, "softplus", seed=31, state_std=0.05, device=DEV),
        make_prefill_inputs([130, 2048, 5], 8, 128, 128, dtype, "uniform", seed=32, state_std=None, device=DEV),
    ]
    for inp in cases:
        (ref_o, ref_s), (out, st, rc) = _run_both(inp)
        assert rc == 0, gdn.status_string(rc)
        assert gdn.gdn_get_device_status() == 0
        assert torch.equal(out, ref_o) and torch.equal(st, ref_s)


def test_noalloc_matches_the_oracle():
    inp = make_prefill_inputs([300, 41], 4, 128, 128, "bf16", "softplus", seed=34, state_std=0.05, device=DEV)
    out = torch.empty_like(inp["v"])
    st = torch.empty((2, 4, 128, 128), device=DEV)
    rc = _noalloc(inp, out, st)
    torch.cuda.synchronize()
    assert rc == 0 and gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle_full(inp)
    eo, es = rel_err(f64(out), o_ref), rel_err(f64(st), s_ref)
    print("noalloc vs oracle: o_err=%.3e s_err=%.3e" % (eo, es))
    assert eo <= TOL[torch.bfloat16] and es <= STATE_TOL_BF16_FP32LEVEL


def test_noalloc_limit_at_its_edge():
    """H = 32, d = 128, one bf16 sequence: the largest length whose workspace fits the scratch runs
    and equals the workspace entry point; one token more is refused before anything is enqueued."""
    H, d = 32, 128
    code = gdn.GDN_BF16
    T_max = _largest_fitting_tokens(H, d, d, code)
    print("largest single-sequence prefill in the scratch: %d tokens (H=%d, d=%d)" % (T_max, H, d))
    assert 1000 < T_max < 8192
    inp = make_prefill_inputs([T_max], H, d, d, "bf16", "softplus", seed=35, device=DEV)
    (ref_o, ref_s), (out, st, rc) = _run_both(inp)
    assert rc == 0, gdn.status_string(rc)
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(st, ref_s)

    big = make_prefill_inputs([T_max + 1], H, d, d, "bf16", "softplus", seed=36, device=DEV)
    assert gdn.workspace_bytes(T_max + 1, 1, H, d, d, code) > SCRATCH_BYTES
    o2 = torch.full_like(big["v"], float("nan"))
    s2 = torch.full((1, H, d, d), float("nan"), device=DEV)
    assert _noalloc(big, o2, s2) == GDN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.isnan(o2.float()).all() and torch.isnan(s2).all()      # nothing was written


def test_noalloc_with_library_normalisation():
    """bf16 | GDN_QK_L2NORM: raw q/k normalised by the library inside the scratch; the same bits as the
    workspace entry point, and a lower size limit (the normalised copies need room)."""
    H, d = 32, 128
    code = gdn.GDN_BF16 | gdn.GDN_QK_L2NORM
    T_norm = _largest_fitting_tokens(H, d, d, code)
    T_plain = _largest_fitting_tokens(H, d, d, gdn.GDN_BF16)
    print("largest normalising prefill in the scratch: %d tokens (plain: %d)" % (T_norm, T_plain))
    assert T_norm < T_plain
    inp = make_prefill_inputs([T_norm], H, d, d, "bf16", "softplus", seed=37, state_std=0.05, device=DEV)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(38)
    sc = torch.exp(torch.empty((T_norm, H, 1), device=DEV).uniform_(-3.0, 3.0, generator=gen))
    inp["q"] = (inp["q"].float() * sc).to(torch.bfloat16)
    inp["k"] = (inp["k"].float() * sc.flip(0)).to(torch.bfloat16)
    (ref_o, ref_s), (out, st, rc) = _run_both(inp, norm=True)
    assert rc == 0, gdn.status_string(rc)
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(st, ref_s)

    # a length that fits without the flag but not with it is refused with it
    mid = make_prefill_inputs([T_norm + 1], H, d, d, "bf16", "softplus", seed=39, device=DEV)
    assert gdn.workspace_bytes(T_norm + 1, 1, H, d, d, gdn.GDN_BF16) <= SCRATCH_BYTES
    o3 = torch.empty_like(mid["v"])
    s3 = torch.empty((1, H, d, d), device=DEV)
    assert _noalloc(mid, o3, s3, norm=True) == GDN_ERR_WORKSPACE
    assert _noalloc(mid, o3, s3, norm=False) == 0
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0


def test_noalloc_refuses_problems_larger_than_its_scratch():
    inp = make_prefill_inputs([64], 2, 64, 64, "bf16", "softplus", seed=33, device=DEV)
    out = torch.empty_like(inp["v"])
    st = torch.empty((1, 2, 64, 64), device=DEV)
    q = inp["q"]
    # claim 131072 tokens over 32 heads: its workspace is far above the 64 MiB scratch, so the call
    # must return GDN_ERR_WORKSPACE before it launches anything
    assert gdn.workspace_bytes(131072, 1, 32, 128, 128) > SCRATCH_BYTES
    rc = gdn.lib().gdn_chunk_prefill_noalloc(_p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["g"]), _p(inp["beta"]),
                                             None, 1, 131072, None, _p(out), _p(st), 32, 128, 128, gdn.GDN_BF16,
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == GDN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
