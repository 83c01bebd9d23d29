"""The entry points are stream-ordered and never synchronise, so they can be
captured in a CUDA graph (with preallocated outputs and workspace) and
replayed; a replay gives exactly the eager results."""
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def test_prefill_and_decode_in_a_cuda_graph():
    from linear_attention_sequence_sm_b200 import gdn
    w = I.custom("graph", batch=2, seq_len=200, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=400, s0_std=0.02)
    x = {k: (v.to(DEV) if v is not None else None) for k, v in I.make_prefill_inputs(w).items()}
    o = torch.empty_like(x["v"])
    sf = torch.empty((2, 4, 128, 128), dtype=torch.float32, device=DEV)
    ws = torch.empty(gdn.workspace_size(gdn.make_shape(x["q"], x["v"])), dtype=torch.uint8, device=DEV)
    dq = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")}
    state = torch.zeros((2, 4, 128, 128), dtype=torch.float32, device=DEV)
    od = torch.empty((2, 4, 128), dtype=torch.bfloat16, device=DEV)

    def work():
        gdn.chunk_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], initial_state=x["initial_state"], out=o,
                          final_state=sf, workspace=ws)
        state.copy_(sf)
        gdn.decode_step(dq["q"], dq["k"], dq["v"], dq["g"], dq["beta"], state, out=od)

    work()  # eager
    torch.cuda.synchronize()
    o_ref, s_ref, od_ref = o.clone(), state.clone(), od.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        work()
    o.zero_(), state.zero_(), od.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(state, s_ref) and torch.equal(od, od_ref)
