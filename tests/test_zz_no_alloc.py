"""gdn_chunk_forward_noalloc: the prefill for callers that cannot allocate.

Callers such as a plugin that its host runtime gives only tensor pointers
(no allocator), or a serving loop that must not call cudaMalloc on the
request path, use this entry point: its scratch is a device array built into
the library instead of a caller-allocated workspace.  This file checks,
through the C ABI, that two calls in a row (the second finding the first
call's leftovers in the shared array) give the same results as
gdn_chunk_forward with a workspace, within the bf16 parity bar, and that a
problem too large for the array is refused before any launch.  The file name
makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu


def _device_inputs(w):
    inp = I.make_prefill_inputs(w)
    dev = torch.device("cuda:0")
    return inp, {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}


def _noalloc_call(gdn, d, chunk):
    """Call gdn_chunk_forward_noalloc directly through ctypes."""
    shape = gdn.make_shape(d["q"], d["v"], d["cu_seqlens"], chunk)
    o = torch.full_like(d["v"], float("nan"))
    sf = torch.full((shape.num_seqs, shape.num_v_heads, shape.head_dim_v, shape.head_dim_k), float("nan"),
                    dtype=torch.float32, device=d["q"].device)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = gdn.LIB.gdn_chunk_forward_noalloc(ctypes.byref(shape), p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]),
                                           p(d["beta"]), p(d["initial_state"]), p(d["cu_seqlens"]), p(o), p(sf),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == gdn.GDN_OK, gdn.LIB.gdn_last_error_message().decode()
    return o, sf


def test_noalloc_matches_workspace_entry_point_twice():
    from linear_attention_sequence_sm_b200 import gdn
    workloads = [
        I.custom("noalloc_varlen", 1, 0, 2, 4, 128, 64, "bf16", seed=61, s0_std=0.02,
                 seq_lens=[130, 1, 64, 0, 257, 33]),
        I.custom("noalloc_batched", batch=3, seq_len=200, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=62),
    ]
    for w in workloads:  # two calls in a row on the shared scratch array
        inp, d = _device_inputs(w)
        o_na, sf_na = _noalloc_call(gdn, d, w.chunk)
        o_ws, sf_ws = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                                        cu_seqlens=d["cu_seqlens"], chunk_size=w.chunk)
        torch.cuda.synchronize()
        eo, es = prefill_errors(inp, o_na, sf_na, to_f64(o_ws), to_f64(sf_ws))
        assert eo <= BAR["bf16"] and es <= BAR["bf16"], (w.name, eo, es)
        assert torch.isfinite(o_na.float()).all() and torch.isfinite(sf_na).all()


def test_noalloc_refuses_too_many_sequences():
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    n = 16385
    q = torch.zeros(1, n, 1, 128, dtype=torch.bfloat16, device=dev)
    v = torch.zeros(1, n, 1, 128, dtype=torch.bfloat16, device=dev)
    cu = torch.arange(n + 1, dtype=torch.int32, device=dev)
    shape = gdn.make_shape(q, v, cu, 64)
    assert shape.num_seqs == n
    st = gdn.LIB.gdn_chunk_forward_noalloc(ctypes.byref(shape), *([None] * 10))
    assert st == gdn.GDN_ERR_UNSUPPORTED
    assert "16384" in gdn.LIB.gdn_last_error_message().decode()
