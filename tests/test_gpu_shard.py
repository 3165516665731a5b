"""Head-sharded layout of one layer on the GPU: each rank's block of heads, run through the library on
its own (here one after another on one GPU, as W ranks would run them side by side), gives the same
bits as the whole layer in one call, and the blocks put back together are that call's output and
final state.  Heads never interact and each head's arithmetic does not depend on H."""
import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.shard import head_range, shard_heads
from linear_attention_10_b200.workloads import make_prefill_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("world", [2, 3, 4])
def test_head_blocks_equal_the_whole_layer(dtype, world):
    inp = make_prefill_inputs([300, 77, 1000], H=8, dk=128, dv=128, dtype=dtype, seed=61, state_std=0.05,
                              device=DEV)
    out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"])
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    for rank in range(world):
        h0, h1 = head_range(rank, world, 8)
        part = shard_heads(inp, rank, world)
        o, s = gdn.gdn_chunk_prefill(part["q"], part["k"], part["v"], part["g"], part["beta"],
                                     cu_seqlens=part["cu_seqlens"], state_in=part["state_in"])
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_status() == 0
        assert torch.equal(o, out[:, h0:h1]) and torch.equal(s, st[:, h0:h1])
