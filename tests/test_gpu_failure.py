"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies gives up,
the kernel records GDN_ERR_TIMEOUT in the status word and returns, and the context stays usable.

gdn_selftest_wait_timeout waits on a barrier that nothing completes -- the same bounded wait the
prefill kernels use on every barrier -- so the test exercises the whole reporting path:
- the wait's time limit;
- the status word;
- gdn_get_device_status reading and clearing it;
- correct results from the next call on the same context.
"""
import time

import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import TOL, f64, oracle_full, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_expired_wait_is_reported_and_the_context_stays_usable():
    L = gdn.lib()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    t0 = time.perf_counter()
    assert L.gdn_selftest_wait_timeout(50_000_000, None) == 0          # a 50 ms limit
    rc = gdn.gdn_get_device_status()
    waited = time.perf_counter() - t0
    assert rc == -7, gdn.status_string(rc)
    assert waited >= 0.045                                             # the wait really ran out
    assert gdn.gdn_get_device_status() == 0                            # reading the word cleared it

    inp = make_prefill_inputs([70, 33], 2, 64, 64, "bf16", "softplus", seed=5, state_std=0.05, device=DEV)
    out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    o_ref, s_ref = oracle_full(inp)
    assert rel_err(f64(out), o_ref) <= TOL[torch.bfloat16] and rel_err(f64(st), s_ref) <= TOL[torch.bfloat16]
