"""GPU parity of the chunkwise prefill (gdn_chunk_forward) against the fp64
oracle, through the C ABI, on seeded synthetic inputs.

Bars: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs, on the max relative L2
error over (sequence, value head) slices of the outputs and of the final
states, and also over (sequence, value head, chunk of 64 tokens) slices of
the outputs, so that one wrong chunk cannot hide inside a long slice.  The
full-size workloads are compared on every unit.
"""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, full_prefill_errors, gpu_prefill, oracle_prefill, prefill_errors

pytestmark = pytest.mark.gpu

# "simt": the fp32 CUDA-core kernel; "default": the single-kernel tensor-core
# path where it applies (the two-kernel one for value heads not a multiple of
# 4); "split": the two-kernel tensor-core path
PATHS = [pytest.param("simt", id="simt"), pytest.param("default", id="default"), pytest.param("split", id="split")]


def _check(w, path, bar=None):
    inp = I.make_prefill_inputs(w)
    o, sf = gpu_prefill(inp, w.chunk, force_simt=path == "simt", split=path == "split")
    r = full_prefill_errors(inp, o, sf, chunk=64)
    bar = bar or BAR[w.dtype]
    print(f"PARITY {w.name} {path}: units {r['units']} o/slice {r['o_slice']:.3e} "
          f"o/chunk {r['o_chunk']:.3e} state {r['state']:.3e} (bar {bar:g})")
    assert r["o_slice"] <= bar and r["o_chunk"] <= bar and r["state"] <= bar, f"{w.name}: {r} (bar {bar:g})"
    return r


def test_tiny_fp32_config():
    """B=1, T=64, 2 q/k and 2 v heads, d=16, C=16, fp32 (bar 1e-4)."""
    _check(I.tiny_fp32(), "default")


@pytest.mark.parametrize("C", [16, 32, 64])
def test_fp32_d128_ragged(C):
    w = I.custom("fp32_d128", batch=2, seq_len=200, hk=2, hv=4, d=128, chunk=C, dtype="f32", seed=21,
                 s0_std=0.02)
    _check(w, "default")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("hk,hv", [(2, 4), (4, 12), (4, 4), (1, 3)])
def test_bf16_d128_c64_batched(path, hk, hv):
    w = I.custom(f"bf16_b2_T300_{hk}x{hv}", batch=2, seq_len=300, hk=hk, hv=hv, d=128, chunk=64, dtype="bf16",
                 seed=22 + hv, s0_std=0.02)
    _check(w, path)


@pytest.mark.parametrize("path", PATHS)
def test_bf16_varlen_edges(path):
    """Ragged lengths around the chunk size, a one-token and an empty sequence,
    per-sequence initial states."""
    w = I.custom("bf16_varlen_edges", 1, 0, 2, 4, 128, 64, "bf16", seed=23, s0_std=0.02,
                 seq_lens=[1, 63, 64, 65, 0, 200, 128, 7])
    _check(w, path)


@pytest.mark.parametrize("path", PATHS)
def test_bf16_mild_decay_long(path):
    """The milder decay of the 4 x 4096 workload (g = -0.1 softplus(N(0,1)+2)),
    where errors have the most room to grow, over 1024 tokens."""
    w = I.custom("bf16_mild", batch=1, seq_len=1024, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=24,
                 g_shift=2.0, g_scale=0.1)
    _check(w, path)


@pytest.mark.parametrize("dk,dv,C,dtype", [(64, 96, 32, "bf16"), (32, 16, 16, "f32"), (128, 64, 64, "f32"),
                                           (8, 128, 16, "bf16")])
def test_other_shapes_simt(dk, dv, C, dtype):
    from parity import to_f64
    from oracle import oracle
    rng = np.random.default_rng(25)
    T, hk, hv = 77, 2, 4
    q = rng.standard_normal((1, T, hk, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((1, T, hk, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, hv, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, T, hv))))
    g = -np.logaddexp(0, rng.standard_normal((1, T, hv)))
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    inp = {"q": torch.tensor(q).to(td), "k": torch.tensor(k).to(td), "v": torch.tensor(v).to(td),
           "g": torch.tensor(g, dtype=torch.float32), "beta": torch.tensor(beta, dtype=torch.float32),
           "initial_state": torch.tensor(0.05 * rng.standard_normal((1, hv, dv, dk)), dtype=torch.float32),
           "cu_seqlens": None}
    o, sf = gpu_prefill(inp, C)
    o_ref, sf_ref = oracle_prefill(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR[dtype] and es <= BAR[dtype], (eo, es)


@pytest.mark.parametrize("path", PATHS)
def test_degenerate_gates(path):
    """beta = 0 on some tokens (pure decay), g far below the kernel floor and
    g = 0 (no decay) on others: the oracle uses them exactly (g = -inf gives
    alpha = 0); the kernels read max(g, -20), a relative change below 1e-8."""
    w = I.custom("bf16_degenerate", batch=1, seq_len=260, hk=1, hv=4, d=128, chunk=64, dtype="bf16", seed=26,
                 s0_std=0.05)
    inp = I.make_prefill_inputs(w)
    inp["beta"][0, 10:40] = 0.0
    inp["g"][0, 50:52] = float("-inf")
    inp["g"][0, 100] = -1e4
    inp["g"][0, 120:180] = 0.0
    o, sf = gpu_prefill(inp, 64, force_simt=path == "simt", split=path == "split")
    o_ref, sf_ref = oracle_prefill(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
    assert torch.isfinite(o.float()).all() and torch.isfinite(sf).all()


@pytest.mark.parametrize("path", PATHS)
def test_no_decay_every_chunk(path):
    """g = 0 on every token (DeltaNet): nothing damps the far entries of the
    chunks' WY factors, so every block of the triangular inverse carries
    weight in the outputs (a decaying input hides a wrong far block)."""
    w = I.custom("bf16_no_decay", batch=2, seq_len=200, hk=1, hv=4, d=128, chunk=64, dtype="bf16", seed=29,
                 s0_std=0.02)
    inp = I.make_prefill_inputs(w)
    inp["g"].zero_()
    o, sf = gpu_prefill(inp, 64, force_simt=path == "simt", split=path == "split")
    r = full_prefill_errors(inp, o, sf, chunk=64)
    print(f"PARITY bf16_no_decay {path}: o/slice {r['o_slice']:.3e} o/chunk {r['o_chunk']:.3e} state {r['state']:.3e}")
    assert r["o_slice"] <= BAR["bf16"] and r["o_chunk"] <= BAR["bf16"] and r["state"] <= BAR["bf16"], r


@pytest.mark.parametrize("path", PATHS)
def test_in_place_state_and_no_final(path):
    """final_state may alias initial_state; output_final_state=False works."""
    from linear_attention_sequence_sm_b200 import gdn
    w = I.custom("bf16_inplace", batch=2, seq_len=130, hk=1, hv=4, d=128, chunk=64, dtype="bf16", seed=27,
                 s0_std=0.02)
    inp = I.make_prefill_inputs(w)
    o_ref, sf_ref = oracle_prefill(inp)
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    state = d["initial_state"].clone()
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=state, final_state=state,
                              chunk_size=64, force_simt=path == "simt", split=path == "split")
    o2, none = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                                 chunk_size=64, output_final_state=False, force_simt=path == "simt",
                                 split=path == "split")
    torch.cuda.synchronize()
    assert none is None and sf.data_ptr() == state.data_ptr()
    eo, es = prefill_errors(inp, o, state, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
    assert torch.equal(o, o2)


def test_bad_cu_seqlens_recorded_not_faulted():
    """Out-of-range cu_seqlens contents are caught on the device: the kernels
    skip their work and the status word reads GDN_ERR_DEVICE_CHECK."""
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    T, hk, hv, d = 100, 1, 4, 128
    q = torch.nn.functional.normalize(torch.randn(1, T, hk, d, device=dev), dim=-1).bfloat16()
    v = torch.randn(1, T, hv, d, device=dev).bfloat16()
    g = -torch.rand(1, T, hv, device=dev)
    b = torch.rand(1, T, hv, device=dev)
    for bad in ([0, 60, 40, 100], [0, 50, 120], [5, 50, 100], [0, 50, 99]):
        cu = torch.tensor(bad, dtype=torch.int32, device=dev)
        shape = gdn.make_shape(q, v, cu, 64)
        ws = torch.zeros(gdn.workspace_size(shape), dtype=torch.uint8, device=dev)
        o = torch.full_like(v, 7.0)
        gdn.chunk_forward(q, q, v, g, b, cu_seqlens=cu, out=o, workspace=ws)
        assert gdn.read_device_status(ws) == gdn.GDN_ERR_DEVICE_CHECK
        assert (o == 7.0).all()
    cu = torch.tensor([0, 50, 100], dtype=torch.int32, device=dev)
    ws = torch.zeros(gdn.workspace_size(gdn.make_shape(q, v, cu, 64)), dtype=torch.uint8, device=dev)
    gdn.chunk_forward(q, q, v, g, b, cu_seqlens=cu, workspace=ws)
    assert gdn.read_device_status(ws) == gdn.GDN_OK


def test_prefill_then_decode_equals_longer_prefill():
    """run(x[:T1]) then decode steps for x[T1:] equals run(x) (oracle too)."""
    from linear_attention_sequence_sm_b200 import gdn
    w = I.custom("bf16_cont", batch=2, seq_len=140, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=28,
                 s0_std=0.02)
    inp = I.make_prefill_inputs(w)
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    T1 = 131
    o1, s = gdn.chunk_forward(d["q"][:, :T1].contiguous(), d["k"][:, :T1].contiguous(),
                              d["v"][:, :T1].contiguous(), d["g"][:, :T1].contiguous(),
                              d["beta"][:, :T1].contiguous(), initial_state=d["initial_state"], chunk_size=64)
    outs = [o1]
    for t in range(T1, w.seq_len):
        outs.append(gdn.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                    d["g"][:, t].contiguous(), d["beta"][:, t].contiguous(), s)[:, None])
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=1)
    o_ref, sf_ref = oracle_prefill(inp)
    eo, es = prefill_errors(inp, o, s, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("path", ["default", "split"])
def test_full_size_prefill_4x4096_all_units(path):
    """The 4 x 4096 token, 16/32-head, d=128, C=64 bf16 workload at full size,
    in the launch configuration the benchmark times (the default path); every
    (sequence, head) unit against the oracle."""
    _check(I.prefill_bf16(), path)


def test_full_size_varlen_all_units():
    """The 32-sequence packed workload (lengths 128..8192, per-sequence
    initial states) at full size, every unit."""
    _check(I.varlen_bf16(), "default")


def test_full_size_long_context_all_units():
    """The 65,536-token, 16/48-head (3 value heads per q/k head), d=128, C=64
    bf16 workload with initial states, at full size, every unit."""
    _check(I.long_bf16(), "default")


def test_path_query_matches_the_launches():
    """gdn_chunk_forward_path names the path the call then takes: one launch
    after the schedule for a single kernel, two for the two-kernel form.  Value
    heads not a multiple of 4 take the two-kernel form with the queried
    workspace and the CUDA-core kernel with only the single-kernel size."""
    import ctypes
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")

    def run(hk, hv, dtype, small=False, **kw):
        w = I.custom(f"path_{hk}_{hv}", batch=1, seq_len=130, hk=hk, hv=hv, d=128, chunk=64, dtype=dtype, seed=71)
        inp = I.make_prefill_inputs(w)
        d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        shape = gdn.make_shape(d["q"], d["v"], None, 64, **kw)
        nbytes = gdn.workspace_size(gdn.make_shape(d["q"], d["v"], None, 64, one_kernel=True)) if small else \
            gdn.workspace_size(shape)
        path = gdn.forward_path(shape, nbytes)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        o = torch.empty_like(d["v"])
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        n0 = gdn.launch_count()
        st = gdn.LIB.gdn_chunk_forward(ctypes.byref(shape), p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]), p(d["beta"]),
                                       None, None, p(o), None, p(ws), nbytes,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        assert st == gdn.GDN_OK and gdn.read_device_status(ws) == gdn.GDN_OK
        assert torch.isfinite(o.float()).all()
        return path, gdn.launch_count() - n0

    assert run(2, 8, "bf16") == ("tc_one_kernel", 2)
    assert run(2, 8, "bf16", split=True) == ("tc_split", 3)
    assert run(2, 6, "bf16") == ("tc_split", 3)
    assert run(2, 6, "bf16", small=True) == ("simt", 2)
    assert run(2, 6, "bf16", one_kernel=True) == ("simt", 2)
    assert run(2, 8, "f32") == ("simt", 2)
    assert run(2, 8, "bf16", force_simt=True) == ("simt", 2)
