"""The allocation-free prefill entry point, called through the C ABI.

gdn_chunk_prefill_noalloc serves callers that cannot allocate device memory when they run a prefill
(an engine that fixes its whole GPU memory plan at start-up, or a latency-critical path where
cudaMalloc could block).  Instead of a caller workspace it uses a fixed scratch array inside the
library.  These checks compare it with gdn_chunk_prefill (caller workspace) on two calls in a row,
so the second call runs on scratch that still holds the first call's contents, and check that a
problem too large for the scratch is refused.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(inp, out, state_out):
    q = inp["q"]
    T, H, dk = q.shape
    dv = inp["v"].shape[2]
    N = inp["cu_seqlens"].numel() - 1
    return gdn.lib().gdn_chunk_prefill_noalloc(
        _p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["g"]), _p(inp["beta"]), _p(inp["cu_seqlens"]), N, T,
        _p(inp["state_in"]), _p(out), _p(state_out), H, dk, dv, gdn.GDN_BF16 if q.dtype == torch.bfloat16 else gdn.GDN_F32,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    cases = [
        make_prefill_inputs([1000, 77, 2500], 8, 128, 128, dtype, "softplus", seed=31, state_std=0.05, device=DEV),
        make_prefill_inputs([130, 2048, 5], 8, 128, 128, dtype, "uniform", seed=32, state_std=None, device=DEV),
    ]
    for inp in cases:
        ref_o, ref_s = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                             cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
        out = torch.full_like(ref_o, float("nan"))
        st = torch.full_like(ref_s, float("nan"))
        rc = _noalloc(inp, out, st)
        assert rc == 0, gdn.status_string(rc)
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_status() == 0
        tol = TOL[inp["q"].dtype]
        assert rel_err(f64(out), f64(ref_o)) <= tol
        assert rel_err(f64(st), f64(ref_s)) <= tol


def test_noalloc_refuses_problems_larger_than_its_scratch():
    inp = make_prefill_inputs([64], 2, 64, 64, "bf16", "softplus", seed=33, device=DEV)
    out = torch.empty_like(inp["v"])
    st = torch.empty((1, 2, 64, 64), device=DEV)
    q = inp["q"]
    # claim 131072 tokens over 32 heads: its workspace is far above the 64 MiB scratch, so the call
    # must return GDN_ERR_WORKSPACE before it launches anything
    assert gdn.workspace_bytes(131072, 1, 32, 128, 128) > (64 << 20)
    rc = gdn.lib().gdn_chunk_prefill_noalloc(_p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["g"]), _p(inp["beta"]),
                                             None, 1, 131072, None, _p(out), _p(st), 32, 128, 128, gdn.GDN_BF16,
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -5
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
