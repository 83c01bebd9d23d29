"""gdn_chunk_forward_noalloc: the prefill for callers that cannot allocate.

Callers such as a plugin that its host runtime gives only tensor pointers
(no allocator), or a serving loop that must not call cudaMalloc on the
request path, use this entry point: its scratch is a device array built into
the library instead of a caller-allocated workspace.  This file checks,
through the C ABI, that two calls in a row (the second finding the first
call's leftovers in the shared array) give exactly the results of
gdn_chunk_forward with a workspace and GDN_FLAG_ONE_KERNEL (both run the same
deterministic kernels on the same inputs), on the tensor-core path and on
the fp32 CUDA-core path,
each after a call with more sequences, and that a problem too large for the
array is refused before any launch.  The file name
makes pytest collect it last.
"""
import ctypes

import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _device_inputs(w):
    inp = I.make_prefill_inputs(w)
    dev = torch.device("cuda:0")
    return inp, {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}


def _noalloc_call(gdn, d, chunk, force_simt=False):
    """Call gdn_chunk_forward_noalloc directly through ctypes."""
    shape = gdn.make_shape(d["q"], d["v"], d["cu_seqlens"], chunk, force_simt)
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
    # (workload, force the fp32 CUDA-core kernel); each call after the first
    # finds fewer sequences than the call before left in the shared array
    cases = [
        (I.custom("noalloc_varlen", 1, 0, 2, 4, 128, 64, "bf16", seed=61, s0_std=0.02,
                  seq_lens=[130, 1, 64, 0, 257, 33]), False),
        (I.custom("noalloc_batched", batch=3, seq_len=200, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=62),
         False),
        (I.custom("noalloc_fp32_d16", batch=2, seq_len=90, hk=2, hv=2, d=16, chunk=16, dtype="f32", seed=63,
                  s0_std=0.05), False),
        (I.custom("noalloc_simt", 1, 0, 1, 3, 128, 64, "bf16", seed=64, s0_std=0.02, seq_lens=[65, 2]), True),
    ]
    for w, simt in cases:  # calls in a row on the shared scratch array
        inp, d = _device_inputs(w)
        o_na, sf_na = _noalloc_call(gdn, d, w.chunk, force_simt=simt)
        o_ws, sf_ws = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                                        cu_seqlens=d["cu_seqlens"], chunk_size=w.chunk, force_simt=simt,
                                        one_kernel=True)
        torch.cuda.synchronize()
        assert torch.equal(o_na, o_ws) and torch.equal(sf_na, sf_ws), w.name
        assert torch.isfinite(o_na.float()).all() and torch.isfinite(sf_na).all()


def test_noalloc_device_status_reads_back():
    """A cu_seqlens rejected on the device shows in the built-in array's status
    word (and the outputs stay unwritten); the next good call clears it."""
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    T, hk, hv, d = 100, 1, 4, 128
    gen = torch.Generator(device="cpu").manual_seed(81)
    q = torch.nn.functional.normalize(torch.randn(1, T, hk, d, generator=gen), dim=-1).bfloat16().to(dev)
    v = torch.randn(1, T, hv, d, generator=gen).bfloat16().to(dev)
    g = (-torch.rand(1, T, hv, generator=gen)).to(dev)
    b = torch.rand(1, T, hv, generator=gen).to(dev)
    bad = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=dev)
    o = torch.full_like(v, 7.0)
    gdn.chunk_forward_noalloc(q, q, v, g, b, cu_seqlens=bad, out=o)
    assert gdn.noalloc_read_device_status(dev) == gdn.GDN_ERR_DEVICE_CHECK
    assert (o == 7.0).all()
    good = torch.tensor([0, 50, 100], dtype=torch.int32, device=dev)
    gdn.chunk_forward_noalloc(q, q, v, g, b, cu_seqlens=good, out=o)
    assert gdn.noalloc_read_device_status(dev) == gdn.GDN_OK
    assert not (o == 7.0).all()


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
