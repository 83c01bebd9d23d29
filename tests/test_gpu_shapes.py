"""Key and value head dims that differ (d_k != d_v) and three value heads per
q/k head, on every path that takes them (the fp32 CUDA-core prefill, decode,
KDA, the multi-token decode, the backward), against the oracle."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def asym_inputs(seed, B, T, hk, hv, dk, dv, dtype, s0_std=0.05):
    """The prefill recipe with d_k != d_v: q, k [B,T,Hk,dk] L2-normalised,
    v [B,T,Hv,dv], g = -softplus(N(0,1)), beta = sigmoid(N(0,1))."""
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    q = I.l2_normalise(I.normal(seed, "aq", (B, T, hk, dk)))
    k = I.l2_normalise(I.normal(seed, "ak", (B, T, hk, dk)))
    v = I.normal(seed, "av", (B, T, hv, dv))
    g = -np.logaddexp(0.0, I.normal(seed, "ag", (B, T, hv)))
    beta = 1.0 / (1.0 + np.exp(-I.normal(seed, "ab", (B, T, hv))))
    s0 = I.normal(seed, "as0", (B, hv, dv, dk), std=s0_std)
    return {"q": torch.from_numpy(q).to(td), "k": torch.from_numpy(k).to(td), "v": torch.from_numpy(v).to(td),
            "g": torch.from_numpy(g).float(), "beta": torch.from_numpy(beta).float(),
            "initial_state": torch.from_numpy(s0).float(), "cu_seqlens": None}


def on_dev(inp):
    return {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 32), (48, 80)])
def test_prefill_f32_asymmetric(dk, dv):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    inp = asym_inputs(500 + dk, 2, 90, 1, 3, dk, dv, "f32")
    d = on_dev(inp)
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                              chunk_size=32)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrent(*(to_f64(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                    initial_state=to_f64(inp["initial_state"]))
    eo, es = prefill_errors(inp, o, sf, o_ref, s_ref)
    assert eo <= BAR["f32"] and es <= BAR["f32"], (eo, es)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_kda_asymmetric(dk, dv):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    inp = asym_inputs(510 + dk, 2, 70, 1, 3, dk, dv, "bf16")
    inp["g"] = torch.from_numpy(-np.logaddexp(0.0, I.normal(511, "akg", (2, 70, 3, dk)))).float()
    d = on_dev(inp)
    o, sf = gdn.kda_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_recurrent(*(to_f64(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                        initial_state=to_f64(inp["initial_state"]))
    eo, es = prefill_errors(inp, o, sf, o_ref, s_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("dv", [64, 96])
def test_decode_multi_other_dv(dv):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    inp = asym_inputs(520 + dv, 4, 3, 1, 3, 128, dv, "bf16")  # 4 sequences x 3 draft tokens
    d = on_dev(inp)
    o, snaps = gdn.decode_multi(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode_multi(*(to_f64(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                       to_f64(inp["initial_state"]))
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(to_f64(o), o_ref) <= BAR["bf16"] and rel(to_f64(snaps), s_ref) <= BAR["bf16"]


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 48)])
def test_backward_asymmetric(dk, dv):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    inp = asym_inputs(530 + dk, 2, 75, 1, 3, dk, dv, "f32")
    dO = torch.from_numpy(I.normal(531, "ado", (2, 75, 3, dv))).float()
    dSf = torch.from_numpy(I.normal(532, "adsf", (2, 3, dv, dk), std=0.1)).float()
    d = on_dev(inp)
    gr = gdn.chunk_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], dO.to(DEV), d_final_state=dSf.to(DEV),
                            initial_state=d["initial_state"])
    torch.cuda.synchronize()
    ref = oracle.backward(*(to_f64(inp[n]) for n in ("q", "k", "v", "g", "beta")), to_f64(dO),
                          dS_final=to_f64(dSf), initial_state=to_f64(inp["initial_state"]))
    rel = lambda a, b: np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    for n, r in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dg", "dg"), ("dbeta", "dbeta"),
                 ("d_initial_state", "dS0")):
        e = rel(to_f64(gr[n]), np.asarray(ref[r]).reshape(gr[n].shape))
        assert e <= 2e-4, (n, e)


def test_decode_generic_asymmetric():
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    inp = asym_inputs(540, 6, 1, 2, 6, 96, 40, "f32")
    d = on_dev(inp)
    st = d["initial_state"].clone()
    o = gdn.decode_step(*(d[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")), st)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode_step(*(to_f64(inp[n][:, 0]) for n in ("q", "k", "v", "g", "beta")),
                                      to_f64(inp["initial_state"]))
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(to_f64(o), o_ref) <= BAR["f32"] and rel(to_f64(st), s_ref) <= BAR["f32"]
