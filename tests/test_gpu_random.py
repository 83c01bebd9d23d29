"""A seeded sweep of random shapes and feature combinations on the GPU
against the oracle: batch or packed varlen (with empty sequences), lengths
from 1 to ~300, 1 to 3 value heads per q/k head, initial states or not, the
input-side flags and the output side, on whichever kernel the shape selects
(the tensor-core kernel needs bf16, d = 128 and Hv a multiple of 4)."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def case(seed):
    rng = np.random.default_rng(seed)
    hk = int(rng.integers(1, 3))
    G = int(rng.integers(1, 4))
    hv = hk * G
    if rng.random() < 0.5:  # make the tensor-core path eligible
        hv = 4 * int(rng.integers(1, 3))
        hk = hv // int(rng.choice([1, 2, 4]))
    d = 128 if rng.random() < 0.7 else int(rng.choice([32, 64]))
    dtype = "bf16" if rng.random() < 0.8 else "f32"
    varlen = rng.random() < 0.5
    if varlen:
        lens = [int(x) for x in rng.integers(0, 160, size=int(rng.integers(1, 5)))]
        B, T = 1, sum(lens)
    else:
        lens, B, T = None, int(rng.integers(1, 4)), int(rng.integers(1, 300))
    return dict(hk=hk, hv=hv, d=d, dtype=dtype, lens=lens, B=B, T=T, s0=bool(rng.random() < 0.6),
                l2=bool(rng.random() < 0.4), logits=bool(rng.random() < 0.4), out=bool(rng.random() < 0.4),
                split=bool(rng.random() < 0.3))


@pytest.mark.parametrize("seed", range(24))
def test_random_prefill(seed):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    c = case(600 + seed)
    if c["T"] == 0:
        pytest.skip("no tokens")
    w = I.custom(f"rand_{seed}", batch=c["B"], seq_len=c["T"], hk=c["hk"], hv=c["hv"], d=c["d"], chunk=64,
                 dtype=c["dtype"], seed=700 + seed, s0_std=0.03 if c["s0"] else 0.0, seq_lens=c["lens"])
    inp = I.make_raw_prefill_inputs(w) if (c["l2"] or c["logits"]) else I.make_prefill_inputs(w)
    if not c["l2"] and (c["logits"]):  # logits only: give unit-norm q, k
        for n in ("q", "k"):
            x = inp[n].float()
            inp[n] = (x / x.norm(dim=-1, keepdim=True)).to(inp[n].dtype)
    if c["l2"] and not c["logits"]:  # normalisation only: give prepared gates
        inp["g"] = torch.nn.functional.logsigmoid(inp["g"])
        inp["beta"] = torch.sigmoid(inp["beta"])
    z = wt = None
    on = None
    if c["out"]:
        z = I.make_output_gate(w)
        wt = I.make_output_weight(w)
        on = gdn.OutputNorm(weight=wt.to(DEV), gate=z.to(DEV), eps=1e-6, activation="silu")
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                              cu_seqlens=d["cu_seqlens"], chunk_size=64, qk_l2norm=c["l2"], gate_logits=c["logits"],
                              output_norm=on, split=c["split"])
    torch.cuda.synchronize()
    q, k, g, b = oracle.prepare_inputs(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["g"]), to_f64(inp["beta"]),
                                       qk_l2norm=c["l2"], gate_logits=c["logits"])
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    o_ref, s_ref = oracle.recurrent(q, k, to_f64(inp["v"]), g, b, initial_state=to_f64(inp["initial_state"]),
                                    cu_seqlens=cu)
    if c["out"]:
        o_ref = oracle.output_side(o_ref, z=to_f64(z), weight=to_f64(wt), eps=1e-6, gate="silu")
    eo, es = prefill_errors(inp, o, sf, o_ref, s_ref)
    bar = BAR[c["dtype"]]
    assert eo <= bar and es <= bar, (c, eo, es)
