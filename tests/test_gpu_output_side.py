"""GPU parity of the mixer's output side done inside the kernels (RMS
normalisation of each (token, value head) output row, a plain, zero-centred
or per-head scale, and a SiLU or sigmoid gate), against the fp64 oracle:
the oracle's recurrence, then its output side, on the same inputs
("Architecture Thread I", "Modern Architecture Improvements"; "Gated
Attention Architectures", the Gated DeltaNet code listing)."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")

# (activation, gate?, weight kind, zero-centred)
CASES = [
    ("silu", True, "shared", False),
    ("sigmoid", True, "per_head", True),
    ("silu", False, None, False),
    ("silu", True, None, True),
]


def out_inputs(seed, rows_shape, hv, dv, dtype, gate, weight, zero_centred):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    z = None
    if gate:
        z = torch.from_numpy(I.normal(seed, "oz", (*rows_shape, hv, dv), std=2.0)).to(td)
    w = None
    if weight == "shared":
        w = torch.from_numpy(I.normal(seed, "ow", (dv,), mean=0.0 if zero_centred else 1.0, std=0.3)).float()
    elif weight == "per_head":
        w = torch.from_numpy(I.normal(seed, "ow", (hv, dv), mean=0.0 if zero_centred else 1.0, std=0.3)).float()
    return z, w


def gpu_norm(z, w, eps, act, zero_centred):
    from linear_attention_sequence_sm_b200 import gdn
    return gdn.OutputNorm(weight=None if w is None else w.to(DEV), gate=None if z is None else z.to(DEV), eps=eps,
                          activation=act, zero_centred=zero_centred)


def oracle_out(o_ref, z, w, eps, act, zero_centred):
    from oracle import oracle
    return oracle.output_side(o_ref, z=to_f64(z), weight=to_f64(w), eps=eps, gate=act, zero_centred=zero_centred)


def prefill_case(inp, chunk, force_simt, z, w, eps, act, zc, **flags):
    from linear_attention_sequence_sm_b200 import gdn
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    y, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                              cu_seqlens=d["cu_seqlens"], chunk_size=chunk, force_simt=force_simt,
                              output_norm=gpu_norm(z, w, eps, act, zc), **flags)
    torch.cuda.synchronize()
    return y, sf


def oracle_prefill_out(inp, z, w, eps, act, zc, qk_l2norm=False, gate_logits=False):
    from oracle import oracle
    q, k, g, b = oracle.prepare_inputs(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["g"]), to_f64(inp["beta"]),
                                       qk_l2norm=qk_l2norm, gate_logits=gate_logits)
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    o_ref, sf_ref = oracle.recurrent(q, k, to_f64(inp["v"]), g, b, initial_state=to_f64(inp["initial_state"]),
                                     cu_seqlens=cu)
    return oracle_out(o_ref, z, w, eps, act, zc), sf_ref


def prefill_inputs(seed, B, T, hk, hv, d, dtype, chunk=64, seq_lens=None, s0_std=0.02):
    w = I.custom(f"out_side_{seed}", batch=B, seq_len=T, hk=hk, hv=hv, d=d, chunk=chunk, dtype=dtype, seed=seed,
                 s0_std=s0_std, seq_lens=seq_lens)
    return I.make_prefill_inputs(w)


@pytest.mark.parametrize("force_simt", [False, True])
@pytest.mark.parametrize("act,gate,weight,zc", CASES)
def test_prefill_bf16_output_side(force_simt, act, gate, weight, zc):
    inp = prefill_inputs(71, B=2, T=300, hk=2, hv=4, d=128, dtype="bf16")
    z, w = out_inputs(72, (2, 300), 4, 128, "bf16", gate, weight, zc)
    y, sf = prefill_case(inp, 64, force_simt, z, w, 1e-6, act, zc)
    y_ref, sf_ref = oracle_prefill_out(inp, z, w, 1e-6, act, zc)
    eo, es = prefill_errors(inp, y, sf, y_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("force_simt", [False, True])
def test_prefill_bf16_output_side_varlen_edges(force_simt):
    """Ragged lengths: the tensor-core kernel's last chunk of a sequence is
    stored row by row, and its gate tile holds the next sequence's rows."""
    lens = [1, 63, 64, 65, 0, 200, 7]
    inp = prefill_inputs(73, B=1, T=sum(lens), hk=1, hv=4, d=128, dtype="bf16", seq_lens=lens)
    z, w = out_inputs(74, (1, sum(lens)), 4, 128, "bf16", True, "shared", False)
    y, sf = prefill_case(inp, 64, force_simt, z, w, 1e-5, "silu", False)
    y_ref, sf_ref = oracle_prefill_out(inp, z, w, 1e-5, "silu", False)
    eo, es = prefill_errors(inp, y, sf, y_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
    assert torch.isfinite(y.float()).all()


def test_prefill_bf16_both_sides():
    """Input side (raw q, k and gate logits) and output side in one call."""
    from test_gpu_input_side import raw_inputs
    inp = raw_inputs(75, B=2, T=200, hk=2, hv=4, d=128, dtype="bf16", s0_std=0.02)
    z, w = out_inputs(76, (2, 200), 4, 128, "bf16", True, "per_head", True)
    y, sf = prefill_case(inp, 64, False, z, w, 1e-6, "silu", True, qk_l2norm=True, gate_logits=True)
    y_ref, sf_ref = oracle_prefill_out(inp, z, w, 1e-6, "silu", True, qk_l2norm=True, gate_logits=True)
    eo, es = prefill_errors(inp, y, sf, y_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("d,C", [(128, 64), (64, 32), (16, 16)])
def test_prefill_f32_output_side(d, C):
    """fp32 inputs take the CUDA-core kernel and its separate output-side
    pass: the 1e-4 bar."""
    inp = prefill_inputs(77, B=1, T=150, hk=2, hv=2, d=d, dtype="f32", chunk=C)
    z, w = out_inputs(78, (1, 150), 2, d, "f32", True, "shared", False)
    y, sf = prefill_case(inp, C, False, z, w, 1e-6, "silu", False)
    y_ref, sf_ref = oracle_prefill_out(inp, z, w, 1e-6, "silu", False)
    eo, es = prefill_errors(inp, y, sf, y_ref, sf_ref)
    assert eo <= BAR["f32"] and es <= BAR["f32"], (eo, es)


def test_prefill_output_side_rows_are_normalised():
    """Without gate or weight, every output row of the tensor-core kernel
    has a root mean square of 1 (up to eps and bf16 rounding)."""
    inp = prefill_inputs(79, B=1, T=256, hk=2, hv=4, d=128, dtype="bf16")
    y, _ = prefill_case(inp, 64, False, None, None, 1e-12, "silu", False)
    rms = y.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2), (rms.min().item(), rms.max().item())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("act,gate,weight,zc", CASES[:2])
def test_decode_output_side(dtype, d, act, gate, weight, zc):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    N, hk, hv, steps = 8, 2, 4, 4
    state0 = I.normal(80, "ds0", (N, hv, d, d), std=0.05)
    state = torch.from_numpy(state0).float().to(DEV)
    ref = state0.copy()
    worst = 0.0
    for t in range(steps):
        x = prefill_inputs(81 + t, B=N, T=1, hk=hk, hv=hv, d=d, dtype=dtype, s0_std=0.0)
        q, k, v = (x[n].reshape(N, -1, d) for n in ("q", "k", "v"))
        g, b = x["g"].reshape(N, hv), x["beta"].reshape(N, hv)
        z, w = out_inputs(90 + t, (N,), hv, d, dtype, gate, weight, zc)
        y = gdn.decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state,
                            output_norm=gpu_norm(z, w, 1e-6, act, zc))
        o_ref, ref = oracle.decode_step(to_f64(q), to_f64(k), to_f64(v), to_f64(g), to_f64(b), ref)
        y_ref = oracle_out(o_ref, z, w, 1e-6, act, zc)
        yg = to_f64(y)
        for n in range(N):
            for h in range(hv):
                worst = max(worst, np.linalg.norm(yg[n, h] - y_ref[n, h]) / np.linalg.norm(y_ref[n, h]))
    torch.cuda.synchronize()
    sg = to_f64(state)
    es = max(np.linalg.norm(sg[n, h] - ref[n, h]) / np.linalg.norm(ref[n, h]) for n in range(N) for h in range(hv))
    assert worst <= BAR[dtype] and es <= BAR[dtype], (worst, es)
