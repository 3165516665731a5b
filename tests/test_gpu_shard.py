"""Head-sharded layout of one layer on the GPU (Ferrite project page, Design section 05: each of the
two machines holds half of every layer).  Each rank's block of heads is run through the library on its
own (here one after another on one GPU, as W ranks would run them side by side) and compared with
the fp64 oracle of those heads at the parity bar; it also gives the same bits as the whole layer in
one call, since heads never interact and each head's arithmetic does not depend on H."""
import numpy as np
import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.shard import head_range, shard_heads
from linear_attention_10_b200.workloads import make_prefill_inputs

from helpers import TOL, f64, oracle_heads, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("world", [2, 3, 4])
def test_head_blocks_match_the_oracle_and_the_whole_layer(dtype, world):
    inp = make_prefill_inputs([300, 77, 1000], H=8, dk=128, dv=128, dtype=dtype, seed=61, state_std=0.05,
                              device=DEV)
    out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    ref = oracle_heads(inp)
    tol = TOL[inp["q"].dtype]
    for rank in range(world):
        h0, h1 = head_range(rank, world, 8)
        part = shard_heads(inp, rank, world)
        o, s = gdn.gdn_chunk_prefill(part["q"], part["k"], part["v"], part["g"], part["beta"],
                                     cu_seqlens=part["cu_seqlens"], state_in=part["state_in"])
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_status() == 0
        # the rank's block against the oracle of its heads
        o_ref = np.stack([ref[h][0] for h in range(h0, h1)], axis=1)
        s_ref = np.stack([ref[h][1] for h in range(h0, h1)], axis=1)
        eo, es = rel_err(f64(o), o_ref), rel_err(f64(s), s_ref)
        print("world=%d rank=%d heads %d..%d: o_err=%.3e s_err=%.3e tol=%g" % (world, rank, h0, h1, eo, es, tol))
        assert eo <= tol and es <= tol
        # and the same bits as the whole layer's call
        assert torch.equal(o, out[:, h0:h1]) and torch.equal(s, st[:, h0:h1])
