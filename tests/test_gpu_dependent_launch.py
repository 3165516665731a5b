"""Back-to-back library calls on one stream equal the same calls separated by synchronisations.

The prep, scan, decode and verify kernels are launched as programmatic dependents of the kernel
before them in the stream: a dependent kernel may become resident while its predecessor is still
running, and must wait for it on the device before reading its results. This test runs a long mixed
sequence of calls with no host synchronisation between them:
- prefills of varying lengths;
- single decode steps;
- chain and tree verifies.

The state is carried from each call into the next, so any read of a result before it is complete
propagates into every later result. Every output and state must equal, bit for bit, the same
sequence run with a device synchronisation after each call (the kernels are deterministic).
"""
import numpy as np
import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import (best_first_parents, make_decode_inputs, make_prefill_inputs,
                                                make_verify_inputs)

pytestmark = pytest.mark.gpu
DEV = "cuda"
N, H, D = 2, 4, 128


def _plan(seed, n_calls=30):
    r = np.random.default_rng(seed)
    calls = []
    for i in range(n_calls):
        kind = ("prefill", "decode", "verify", "tree")[int(r.integers(0, 4))]
        if kind == "prefill":
            lens = [int(r.integers(1, 300)) for _ in range(N)]
            calls.append((kind, make_prefill_inputs(lens, H=H, dk=D, dv=D, dtype="bf16", seed=1000 + i,
                                                    device=DEV)))
        elif kind == "decode":
            calls.append((kind, make_decode_inputs(N, H, D, D, 1, dtype="bf16", seed=2000 + i, device=DEV)))
        else:
            Tk = int(r.integers(2, 7))
            d = make_verify_inputs(N, H, D, D, Tk, dtype="bf16", seed=3000 + i, device=DEV)
            d["parents"] = torch.tensor([best_first_parents(Tk)] * N, dtype=torch.int32, device=DEV)
            calls.append((kind, d))
    torch.cuda.synchronize()
    return calls


def _run(calls, state0, sync):
    """Runs the calls in order; returns every output and the state after every call."""
    state = state0.clone()
    results = []
    for kind, d in calls:
        if kind == "prefill":
            out, st = gdn.gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], cu_seqlens=d["cu_seqlens"],
                                            state_in=state)
            results.append(out)
            state = st
        elif kind == "decode":
            out = gdn.gdn_decode_step(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], state)
            results.append(out)
        else:
            if kind == "verify":
                out, sts = gdn.gdn_decode_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], state)
            else:
                out, sts = gdn.gdn_decode_verify_tree(d["q"], d["k"], d["v"], d["g"], d["beta"], d["parents"],
                                                      state)
            results.append(out)
            state = sts[:, -1].contiguous()                     # continue from the last drafted token
        results.append(state.clone())
        if sync:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    return results


@pytest.mark.parametrize("seed", [1, 2])
def test_back_to_back_calls_equal_synchronised_calls(seed):
    calls = _plan(seed)
    state0 = torch.randn((N, H, D, D), device=DEV) * 0.05
    ref = _run(calls, state0, sync=True)
    assert gdn.gdn_get_device_status() == 0
    for _ in range(3):
        got = _run(calls, state0, sync=False)
        assert gdn.gdn_get_device_status() == 0
        assert len(got) == len(ref)
        for i, (a, b) in enumerate(zip(got, ref)):
            assert torch.equal(a, b), "result %d (call %d, %s) differs" % (i, i // 2, calls[i // 2][0])
