"""GPU parity of the input side's short causal convolution (gdn_short_conv)
against the fp64 oracle ("Architecture Thread I", "Modern Architecture
Improvements": projection -> short conv -> SiLU).  The conv states are
copies of inputs, so they must match exactly; outputs meet the dtype's bar
per (sequence, channel group) slice."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


def conv_case(seed, lead, ch, W, dtype, lens=None, with_state=True):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.from_numpy(I.normal(seed, "cx", (*lead, *ch))).to(td)
    w = torch.from_numpy(I.normal(seed, "cw", (*ch, W), std=1.0 / np.sqrt(W))).float()
    n = len(lens) if lens is not None else lead[0]
    st = torch.from_numpy(I.normal(seed, "cs", (n, *ch, W - 1))).float() if with_state else None
    cu = None
    if lens is not None:
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return x, w, st, cu


def run_both(x, w, st, cu, silu=True):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    y, so = gdn.short_conv(x.to(DEV), w.to(DEV), cu_seqlens=None if cu is None else cu.to(DEV),
                           state=None if st is None else st.to(DEV), silu=silu)
    torch.cuda.synchronize()
    y_ref, s_ref = oracle.short_conv(to_f64(x), to_f64(w), cu_seqlens=None if cu is None else cu.numpy(),
                                     state=to_f64(st), silu=silu)
    return to_f64(y), to_f64(so), y_ref, s_ref


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_conv_batched(dtype, W):
    x, w, st, cu = conv_case(40 + W, (3, 200), (2, 128), W, dtype)
    y, so, y_ref, s_ref = run_both(x, w, st, cu)
    assert rel(y, y_ref) <= BAR[dtype], rel(y, y_ref)
    assert np.array_equal(so, s_ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_state", [False, True])
def test_conv_varlen_edges(dtype, with_state):
    """Empty sequences, sequences shorter than W - 1, and the boundaries of the
    threads' token groups
    inside and between sequences; 16 heads of 128 (several channel groups)."""
    lens = [0, 1, 2, 63, 64, 65, 0, 130, 3, 200]
    x, w, st, cu = conv_case(50, (sum(lens),), (16, 128), 4, dtype, lens=lens, with_state=with_state)
    y, so, y_ref, s_ref = run_both(x, w, st, cu)
    cuv = cu.numpy()
    for n in range(len(lens)):
        a, b = cuv[n], cuv[n + 1]
        if b > a:
            assert rel(y[a:b], y_ref[a:b]) <= BAR[dtype], (n, rel(y[a:b], y_ref[a:b]))
    assert np.array_equal(so, s_ref)
    y2, _, y2_ref, _ = run_both(x, w, st, cu, silu=False)
    assert rel(y2, y2_ref) <= BAR[dtype]


def test_conv_continuation_on_gpu():
    """A sequence split in two, the second part started from the first
    part's conv state, equals the unsplit call."""
    from linear_attention_sequence_sm_b200 import gdn
    x, w, st, _ = conv_case(60, (1, 300), (4, 64), 4, "f32")
    xd, wd, sd = x.to(DEV), w.to(DEV), st.to(DEV)
    y, s = gdn.short_conv(xd, wd, state=sd)
    y1, s1 = gdn.short_conv(xd[:, :131].contiguous(), wd, state=sd)
    y2, s2 = gdn.short_conv(xd[:, 131:].contiguous(), wd, state=s1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], dim=1), y) and torch.equal(s2, s)


def test_conv_full_size_q():
    """The 4 x 4096 workload's q tensor ([4, 4096, 16, 128] bf16), W = 4."""
    w_ = I.prefill_bf16()
    q = I.make_prefill_inputs(w_)["q"]
    wt = torch.from_numpy(I.normal(70, "cw", (16, 128, 4), std=0.5)).float()
    y, so, y_ref, s_ref = run_both(q, wt, None, None)
    worst = max(rel(y[b, :, h], y_ref[b, :, h]) for b in range(4) for h in range(16))
    assert worst <= BAR["bf16"], worst
    assert np.array_equal(so, s_ref)


def test_conv_then_prefill_matches_composed_oracle():
    """The whole input side on the GPU -- the convolutions with SiLU here,
    the L2 normalisation of q and k inside the tensor-core prefill
    (GDN_FLAG_QK_L2NORM) -- against the oracle's composed input side and its
    recurrence."""
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    B, T, hk, hv, d, W = 2, 150, 2, 4, 128, 4
    w_ = I.custom("conv_e2e", batch=B, seq_len=T, hk=hk, hv=hv, d=d, chunk=64, dtype="bf16", seed=80, s0_std=0.02)
    raw = I.make_raw_prefill_inputs(w_)
    wq, wk = (torch.from_numpy(I.normal(81, t, (hk, d, W), std=0.5)).float() for t in ("wq", "wk"))
    wv = torch.from_numpy(I.normal(81, "wv", (hv, d, W), std=0.5)).float()
    g = torch.nn.functional.logsigmoid(raw["g"])
    b = torch.sigmoid(raw["beta"])
    dq, dk, dv = (gdn.short_conv(raw[n].to(DEV), wt.to(DEV))[0] for n, wt in (("q", wq), ("k", wk), ("v", wv)))
    o, sf = gdn.chunk_forward(dq, dk, dv, g.to(DEV), b.to(DEV), initial_state=raw["initial_state"].to(DEV),
                              qk_l2norm=True)
    torch.cuda.synchronize()
    qn, kn, vc, _ = oracle.conv_input_side(to_f64(raw["q"]), to_f64(raw["k"]), to_f64(raw["v"]), to_f64(wq),
                                           to_f64(wk), to_f64(wv))
    o_ref, s_ref = oracle.recurrent(qn, kn, vc, to_f64(g), to_f64(b), initial_state=to_f64(raw["initial_state"]))
    og, sg = to_f64(o), to_f64(sf)
    eo = max(rel(og[n, :, h], o_ref[n, :, h]) for n in range(B) for h in range(hv))
    es = max(rel(sg[n, h], s_ref[n, h]) for n in range(B) for h in range(hv))
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)
