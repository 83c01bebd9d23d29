"""GPU parity of Kimi Delta Attention (one decay per key channel;
"Gated Attention Architectures", section 8) against the fp64 oracle's KDA
recurrence: prefill (bf16 and fp32, batched and packed, start states, the
input and output sides) and decode."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def kda_inputs(seed, B, T, hk, hv, d, dtype, seq_lens=None, s0_std=0.02, g_scale=1.0):
    w = I.custom(f"kda_{seed}", batch=B, seq_len=T, hk=hk, hv=hv, d=d, chunk=64, dtype=dtype, seed=seed,
                 s0_std=s0_std, seq_lens=seq_lens, g_scale=g_scale)
    inp = I.make_prefill_inputs(w)
    inp["g"] = I.make_kda_gates(w)
    return inp


def gpu_kda(inp, **kw):
    from linear_attention_sequence_sm_b200 import gdn
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    o, sf = gdn.kda_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                            cu_seqlens=d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o, sf


def oracle_kda(inp, qk_l2norm=False, gate_logits=False):
    from oracle import oracle
    q, k, g, b = oracle.prepare_kda_inputs(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["g"]),
                                           to_f64(inp["beta"]), qk_l2norm=qk_l2norm, gate_logits=gate_logits)
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    return oracle.kda_recurrent(q, k, to_f64(inp["v"]), g, b, initial_state=to_f64(inp["initial_state"]),
                                cu_seqlens=cu)


@pytest.mark.parametrize("g_scale", [1.0, 0.05])
def test_kda_prefill_bf16(g_scale):
    inp = kda_inputs(101, B=2, T=300, hk=2, hv=4, d=128, dtype="bf16", g_scale=g_scale)
    o, sf = gpu_kda(inp)
    o_ref, sf_ref = oracle_kda(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("d", [128, 64, 16, 100])
def test_kda_prefill_f32(d):
    inp = kda_inputs(102, B=1, T=150, hk=2, hv=2, d=d, dtype="f32", s0_std=0.05)
    o, sf = gpu_kda(inp)
    o_ref, sf_ref = oracle_kda(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["f32"] and es <= BAR["f32"], (eo, es)


def test_kda_prefill_varlen_edges():
    lens = [1, 63, 64, 65, 0, 200, 7]
    inp = kda_inputs(103, B=1, T=sum(lens), hk=1, hv=4, d=128, dtype="bf16", seq_lens=lens)
    o, sf = gpu_kda(inp)
    o_ref, sf_ref = oracle_kda(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
    assert torch.equal(sf[4], inp["initial_state"][4].to(DEV))  # the empty sequence keeps its state


def test_kda_scalar_decay_matches_gdn_on_gpu():
    """With the same decay on every channel, the KDA kernel and the gated
    delta rule kernels agree (different algorithms: rounding only)."""
    from linear_attention_sequence_sm_b200 import gdn
    inp = kda_inputs(104, B=2, T=256, hk=2, hv=4, d=128, dtype="bf16")
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    g_scalar = d["g"][..., 0].contiguous()
    g_rep = g_scalar[..., None].expand_as(d["g"]).contiguous()
    o1, s1 = gdn.kda_forward(d["q"], d["k"], d["v"], g_rep, d["beta"], initial_state=d["initial_state"])
    o2, s2 = gdn.chunk_forward(d["q"], d["k"], d["v"], g_scalar, d["beta"], initial_state=d["initial_state"])
    torch.cuda.synchronize()
    rel = lambda x, y: float((x.float() - y.float()).norm() / y.float().norm())
    assert rel(o1, o2) < 1e-2 and rel(s1, s2) < 1e-2, (rel(o1, o2), rel(s1, s2))


def test_kda_prefill_input_and_output_sides():
    """Raw q, k and per-channel decay logits, with the output side."""
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    from test_gpu_input_side import raw_inputs
    inp = raw_inputs(105, B=2, T=200, hk=2, hv=4, d=128, dtype="bf16", s0_std=0.02)
    inp["g"] = torch.from_numpy(I.normal(105, "kda_logit", (2, 200, 4, 128), mean=2.0)).float()
    z = torch.from_numpy(I.normal(106, "kda_z", (2, 200, 4, 128), std=2.0)).to(torch.bfloat16)
    w = torch.from_numpy(I.normal(106, "kda_w", (128,), mean=1.0, std=0.2)).float()
    on = gdn.OutputNorm(weight=w.to(DEV), gate=z.to(DEV), eps=1e-6, activation="silu")
    o, sf = gpu_kda(inp, qk_l2norm=True, gate_logits=True, output_norm=on)
    o_ref, sf_ref = oracle_kda(inp, qk_l2norm=True, gate_logits=True)
    y_ref = oracle.output_side(o_ref, z=to_f64(z), weight=to_f64(w), eps=1e-6, gate="silu")
    eo, es = prefill_errors(inp, o, sf, y_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("with_out", [False, True])
def test_kda_decode(dtype, d, with_out):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    N, hk, hv, steps = 8, 2, 4, 5
    state0 = I.normal(110, "kds0", (N, hv, d, d), std=0.05)
    state = torch.from_numpy(state0).float().to(DEV)
    ref = state0.copy()
    worst = 0.0
    for t in range(steps):
        x = kda_inputs(111 + t, B=N, T=1, hk=hk, hv=hv, d=d, dtype=dtype, s0_std=0.0)
        q, k, v = (x[n].reshape(N, -1, d) for n in ("q", "k", "v"))
        g, b = x["g"].reshape(N, hv, d), x["beta"].reshape(N, hv)
        on, z, wt = None, None, None
        if with_out:
            z = torch.from_numpy(I.normal(120 + t, "kz", (N, hv, d), std=2.0)).to(q.dtype)
            wt = torch.from_numpy(I.normal(120 + t, "kw", (d,), mean=1.0, std=0.2)).float()
            on = gdn.OutputNorm(weight=wt.to(DEV), gate=z.to(DEV), eps=1e-6, activation="sigmoid")
        y = gdn.kda_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state, output_norm=on)
        o_ref, ref = oracle.kda_decode_step(to_f64(q), to_f64(k), to_f64(v), to_f64(g), to_f64(b), ref)
        if with_out:
            o_ref = oracle.output_side(o_ref, z=to_f64(z), weight=to_f64(wt), eps=1e-6, gate="sigmoid")
        yg = to_f64(y)
        for n in range(N):
            for h in range(hv):
                worst = max(worst, np.linalg.norm(yg[n, h] - o_ref[n, h]) / np.linalg.norm(o_ref[n, h]))
    torch.cuda.synchronize()
    sg = to_f64(state)
    es = max(np.linalg.norm(sg[n, h] - ref[n, h]) / np.linalg.norm(ref[n, h]) for n in range(N) for h in range(hv))
    assert worst <= BAR[dtype] and es <= BAR[dtype], (worst, es)


def test_kda_tensor_core_path_is_taken_and_matches_token_order():
    """bf16, d = 128, C = 64 runs the tensor-core chunkwise form (its own launch
    count: schedule, factors, chunk loop); the token-order kernel
    (force_simt) agrees within rounding, and both meet the oracle."""
    from linear_attention_sequence_sm_b200 import gdn
    inp = kda_inputs(130, B=2, T=200, hk=2, hv=4, d=128, dtype="bf16")
    n0 = gdn.launch_count()
    o, sf = gpu_kda(inp)
    assert gdn.launch_count() - n0 == 3
    o2, sf2 = gpu_kda(inp, force_simt=True)
    o_ref, sf_ref = oracle_kda(inp)
    for oo, ss in ((o, sf), (o2, sf2)):
        eo, es = prefill_errors(inp, oo, ss, o_ref, sf_ref)
        assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("strong", [1, 40])
def test_kda_tensor_core_strongly_decaying_channels(strong):
    """Channels whose decay over a chunk passes e^-80 (here 3 per token for 64
    tokens) leave the factorised Gram and are added with their exact
    exponents; a few of them, and most of them."""
    inp = kda_inputs(131, B=1, T=260, hk=1, hv=2, d=128, dtype="bf16")
    g = inp["g"].clone()
    g[..., :strong] = -3.0
    inp["g"] = g
    o, sf = gpu_kda(inp)
    o_ref, sf_ref = oracle_kda(inp)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


def test_kda_tensor_core_full_size_all_units():
    """The 4 x 4096 prefill workload with per-channel decays, every (sequence,
    value head) unit against the oracle, per slice and per 64-token chunk."""
    from parity import full_prefill_errors
    w = I.prefill_bf16()
    inp = I.make_prefill_inputs(w)
    inp["g"] = I.make_kda_gates(w)
    o, sf = gpu_kda(inp)
    err = full_prefill_errors(inp, o, sf, kda=True)
    print(f"PARITY kda {w.name}: units {err['units']} o/slice {err['o_slice']:.3e} o/chunk {err['o_chunk']:.3e} "
          f"state {err['state']:.3e}")
    assert err["o_slice"] <= BAR["bf16"] and err["o_chunk"] <= BAR["bf16"] and err["state"] <= BAR["bf16"], err
