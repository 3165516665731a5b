"""The prefill on a side stream, back to back with the call that feeds it, and inside a CUDA graph;
a chain of decode steps and a tree verify inside a CUDA graph.

The prep, scan, decode and verify kernels are launched as programmatic dependents of the kernel
before them in the stream, and wait for it on the device before reading its results. These checks
confirm that the dependency holds in the ways a caller uses the library:
- on a non-default stream;
- two calls in a row where the second resumes from the first's final state, with nothing between
  them on the host;
- recorded into a CUDA graph and replayed.

Each result must be identical, bit for bit, to the same call run eagerly on the default stream
with a synchronisation after it.
"""
import pytest
import torch

from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENS = [300, 77, 1000]


def _inputs(dtype, seed, lens=LENS):
    return make_prefill_inputs(lens, H=4, dk=128, dv=128, dtype=dtype, seed=seed, state_std=0.05, device=DEV)


def _eager(inp, state_in=None):
    out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    cu_seqlens=inp["cu_seqlens"],
                                    state_in=inp["state_in"] if state_in is None else state_in)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    return out.clone(), st.clone()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_side_stream_matches_default_stream(dtype):
    inp = _inputs(dtype, 11)
    ref_out, ref_st = _eager(inp)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out, st = gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                        cu_seqlens=inp["cu_seqlens"], state_in=inp["state_in"], stream=s)
    s.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(out, ref_out) and torch.equal(st, ref_st)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_back_to_back_calls_feed_each_other(dtype):
    """Call 2 reads call 1's final state as its initial state, launched right after call 1."""
    a, b = _inputs(dtype, 21), _inputs(dtype, 22)
    ref1_out, ref1_st = _eager(a)
    ref2_out, ref2_st = _eager(b, state_in=ref1_st)
    out1, st1 = gdn.gdn_chunk_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=a["cu_seqlens"],
                                      state_in=a["state_in"])
    out2, st2 = gdn.gdn_chunk_prefill(b["q"], b["k"], b["v"], b["g"], b["beta"], cu_seqlens=b["cu_seqlens"],
                                      state_in=st1)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    assert torch.equal(out1, ref1_out) and torch.equal(st1, ref1_st)
    assert torch.equal(out2, ref2_out) and torch.equal(st2, ref2_st)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_cuda_graph_replay_matches_eager(dtype):
    inp = _inputs(dtype, 31)
    ref_out, ref_st = _eager(inp)
    T, H, dk = inp["q"].shape
    N = inp["cu_seqlens"].numel() - 1
    code = gdn.GDN_BF16 if inp["q"].dtype == torch.bfloat16 else gdn.GDN_F32
    ws = torch.empty(gdn.workspace_bytes(T, N, H, dk, dk, code), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(ref_out)
    st = torch.empty_like(ref_st)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # one eager call on the capture stream first (kernel attributes, tensor maps, status word)
        gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                              state_in=inp["state_in"], out=out, state_out=st, workspace=ws, stream=s)
    s.synchronize()
    out.zero_()
    st.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                              state_in=inp["state_in"], out=out, state_out=st, workspace=ws,
                              stream=torch.cuda.current_stream())
    for _ in range(3):
        out.zero_()
        st.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_status() == 0
        assert torch.equal(out, ref_out) and torch.equal(st, ref_st)
    del graph


def test_decode_chain_and_tree_verify_graph_replay_matches_eager():
    """Eight chained decode steps and a tree verify recorded into one CUDA graph: each replay
    equals the eager sequence bit for bit (the decode and verify kernels are dependent launches)."""
    from linear_attention_10_b200.workloads import best_first_parents, make_decode_inputs, make_verify_inputs
    B, H, d, steps = 4, 3, 128, 8
    dd = make_decode_inputs(B, H, d, d, steps, dtype="bf16", seed=41, device=DEV)
    vd = make_verify_inputs(B, H, d, d, 6, dtype="bf16", seed=42, device=DEV)
    par = torch.tensor([best_first_parents(6)] * B, dtype=torch.int32, device=DEV)

    def sequence(S, outs, vout, vst, stream=None):
        for t in range(steps):
            gdn.gdn_decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["g"][t], dd["beta"][t], S, out=outs[t],
                                stream=stream)
        gdn.gdn_decode_verify_tree(vd["q"], vd["k"], vd["v"], vd["g"], vd["beta"], par, S, states_out=vst,
                                   out=vout, stream=stream)

    def buffers():
        return (dd["state"].clone(), [torch.empty((B, H, d), dtype=torch.bfloat16, device=DEV) for _ in range(steps)],
                torch.empty((B, 6, H, d), dtype=torch.bfloat16, device=DEV),
                torch.empty((B, 6, H, d, d), dtype=torch.float32, device=DEV))

    S_ref, o_ref, vo_ref, vs_ref = buffers()
    sequence(S_ref, o_ref, vo_ref, vs_ref)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0

    S, outs, vout, vst = buffers()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        sequence(S, outs, vout, vst, stream=torch.cuda.current_stream())
    for _ in range(2):
        S.copy_(dd["state"])
        graph.replay()
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_status() == 0
        assert torch.equal(S, S_ref) and torch.equal(vout, vo_ref) and torch.equal(vst, vs_ref)
        assert all(torch.equal(a, b) for a, b in zip(outs, o_ref))
    del graph
