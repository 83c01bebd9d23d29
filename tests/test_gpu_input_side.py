"""GPU parity of the mixer's input side done inside the kernels
(GDN_FLAG_QK_L2NORM: raw q and k normalised per head; GDN_FLAG_GATE_LOGITS:
g and beta given as the decay and write logits), against the fp64 oracle on
the same raw inputs prepared in fp64 ("Gated Attention Architectures", the
Gated DeltaNet code listing; "Architecture Thread I", "Modern Architecture
Improvements")."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, prefill_errors, to_f64

pytestmark = pytest.mark.gpu


def raw_inputs(seed, B, T, hk, hv, d, dtype, seq_lens=None, s0_std=0.0):
    """Raw projections: q and k rows N(0,1) times a per-row norm spread over
    [0.3, 6]; decay logits N(1.5, 1) (mild decay), write logits N(0, 1)."""
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    rows = B * T
    q = I.normal(seed, "rq", (rows, hk, d)) * (0.3 + 5.7 * I.uniform(seed, "rqs", rows * hk).reshape(rows, hk, 1))
    k = I.normal(seed, "rk", (rows, hk, d)) * (0.3 + 5.7 * I.uniform(seed, "rks", rows * hk).reshape(rows, hk, 1))
    v = I.normal(seed, "rv", (rows, hv, d))
    a = I.normal(seed, "ra", (rows, hv), mean=1.5)
    b = I.normal(seed, "rb", (rows, hv))
    shp = (B, T)
    out = {
        "q": torch.from_numpy(q.reshape(*shp, hk, d)).to(td),
        "k": torch.from_numpy(k.reshape(*shp, hk, d)).to(td),
        "v": torch.from_numpy(v.reshape(*shp, hv, d)).to(td),
        "g": torch.from_numpy(a.reshape(*shp, hv)).float(),
        "beta": torch.from_numpy(b.reshape(*shp, hv)).float(),
        "initial_state": None,
        "cu_seqlens": None,
    }
    n = len(seq_lens) if seq_lens is not None else B
    if s0_std > 0:
        out["initial_state"] = torch.from_numpy(I.normal(seed, "rs0", (n, hv, d, d), std=s0_std)).float()
    if seq_lens is not None:
        out["cu_seqlens"] = torch.from_numpy(np.concatenate([[0], np.cumsum(seq_lens)]).astype(np.int32))
    return out


def oracle_raw(inp, qk_l2norm, gate_logits):
    from oracle import oracle
    q, k, g, b = oracle.prepare_inputs(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["g"]), to_f64(inp["beta"]),
                                       qk_l2norm=qk_l2norm, gate_logits=gate_logits)
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    return oracle.recurrent(q, k, to_f64(inp["v"]), g, b, initial_state=to_f64(inp["initial_state"]),
                            cu_seqlens=cu)


def gpu_raw(inp, chunk, qk_l2norm, gate_logits, path="default"):
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                              cu_seqlens=d["cu_seqlens"], chunk_size=chunk, force_simt=path == "simt",
                              split=path == "split", qk_l2norm=qk_l2norm, gate_logits=gate_logits)
    torch.cuda.synchronize()
    return o, sf


PATHS = ["default", "split", "simt"]  # one-kernel tensor-core, two-kernel tensor-core, fp32 CUDA cores


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("qk_l2norm,gate_logits", [(True, True), (True, False), (False, True)])
def test_prefill_bf16_raw_inputs(path, qk_l2norm, gate_logits):
    inp = raw_inputs(61, B=2, T=300, hk=2, hv=4, d=128, dtype="bf16", s0_std=0.02)
    if not qk_l2norm:  # the caller normalised q and k
        for n in ("q", "k"):
            x = inp[n].float()
            inp[n] = (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    if not gate_logits:  # the caller gave g <= 0 and beta in (0, 1)
        inp["g"] = torch.nn.functional.logsigmoid(inp["g"])
        inp["beta"] = torch.sigmoid(inp["beta"])
    o, sf = gpu_raw(inp, 64, qk_l2norm, gate_logits, path)
    o_ref, sf_ref = oracle_raw(inp, qk_l2norm, gate_logits)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


@pytest.mark.parametrize("path", PATHS)
def test_prefill_bf16_raw_varlen_edges(path):
    """Ragged lengths (1, 63, 64, 65, 0, 200, 7): padded rows of a chunk carry
    the next sequence's raw rows or zeros, and must not reach any output."""
    lens = [1, 63, 64, 65, 0, 200, 7]
    inp = raw_inputs(62, B=1, T=sum(lens), hk=1, hv=4, d=128, dtype="bf16", seq_lens=lens, s0_std=0.02)
    o, sf = gpu_raw(inp, 64, True, True, path)
    o_ref, sf_ref = oracle_raw(inp, True, True)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
    assert torch.isfinite(o.float()).all() and torch.isfinite(sf).all()


@pytest.mark.parametrize("d,C", [(128, 64), (64, 32), (16, 16)])
def test_prefill_f32_raw_inputs(d, C):
    """fp32 inputs take the CUDA-core kernel: the 1e-4 bar."""
    inp = raw_inputs(63, B=1, T=150, hk=2, hv=2, d=d, dtype="f32", s0_std=0.05)
    o, sf = gpu_raw(inp, C, True, True)
    o_ref, sf_ref = oracle_raw(inp, True, True)
    eo, es = prefill_errors(inp, o, sf, o_ref, sf_ref)
    assert eo <= BAR["f32"] and es <= BAR["f32"], (eo, es)


def test_prefill_raw_equals_prepared_on_gpu():
    """The fused input side agrees with the same path fed inputs prepared
    by torch on the GPU (different rounding order only)."""
    from linear_attention_sequence_sm_b200 import gdn
    inp = raw_inputs(64, B=2, T=256, hk=2, hv=4, d=128, dtype="bf16")
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o1, s1 = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], qk_l2norm=True, gate_logits=True)
    qn = torch.nn.functional.normalize(d["q"].float(), dim=-1).to(torch.bfloat16)
    kn = torch.nn.functional.normalize(d["k"].float(), dim=-1).to(torch.bfloat16)
    o2, s2 = gdn.chunk_forward(qn, kn, d["v"], torch.nn.functional.logsigmoid(d["g"]), torch.sigmoid(d["beta"]))
    torch.cuda.synchronize()
    rel = lambda x, y: float((x.float() - y.float()).norm() / y.float().norm())
    assert rel(o1, o2) < 1.5e-2 and rel(s1, s2) < 1.5e-2, (rel(o1, o2), rel(s1, s2))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 64])
def test_decode_raw_inputs(dtype, d):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    N, hk, hv, steps = 8, 2, 4, 6
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    dev = torch.device("cuda:0")
    state0 = I.normal(65, "ds0", (N, hv, d, d), std=0.05)
    state = torch.from_numpy(state0).float().to(dev)
    ref = state0.copy()
    worst = 0.0
    for t in range(steps):
        x = raw_inputs(66 + t, B=N, T=1, hk=hk, hv=hv, d=d, dtype=dtype)
        q, k, v = (x[n].reshape(N, -1, d) for n in ("q", "k", "v"))
        a, b = x["g"].reshape(N, hv), x["beta"].reshape(N, hv)
        o = gdn.decode_step(q.to(dev), k.to(dev), v.to(dev), a.to(dev), b.to(dev), state,
                            qk_l2norm=True, gate_logits=True)
        qp, kp, gp, bp = oracle.prepare_inputs(to_f64(q), to_f64(k), to_f64(a), to_f64(b),
                                               qk_l2norm=True, gate_logits=True)
        o_ref, ref = oracle.decode_step(qp, kp, to_f64(v), gp, bp, ref)
        og = to_f64(o)
        for n in range(N):
            for h in range(hv):
                worst = max(worst, np.linalg.norm(og[n, h] - o_ref[n, h]) / np.linalg.norm(o_ref[n, h]))
    torch.cuda.synchronize()
    sg = to_f64(state)
    es = max(np.linalg.norm(sg[n, h] - ref[n, h]) / np.linalg.norm(ref[n, h]) for n in range(N) for h in range(hv))
    assert worst <= BAR[dtype] and es <= BAR[dtype], (worst, es)
