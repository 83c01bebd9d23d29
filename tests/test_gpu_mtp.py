"""GPU parity of the multi-token decode used to verify draft tokens
(several tokens per sequence in one pass, with the state after every token;
"Architecture Thread I", the Qwen3-Next passage on multi-token prediction)
and of the commit of an accepted prefix, against the oracle's decode step
applied token by token."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, to_f64

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def mtp_inputs(seed, N, K, hk, hv, d, dtype):
    w = I.custom(f"mtp_{seed}", batch=N, seq_len=K, hk=hk, hv=hv, d=d, chunk=64, dtype=dtype, seed=seed)
    return I.make_prefill_inputs(w)  # [N, K, H, d] = N sequences of K draft tokens


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 3, 8, 16])
def test_decode_multi_parity(dtype, K):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    N, hk, hv, d = 6, 2, 4, 128
    x = mtp_inputs(200 + K, N, K, hk, hv, d, dtype)
    state0 = I.normal(201, "mtp_s0", (N, hv, d, d), std=0.05)
    state = torch.from_numpy(state0).float().to(DEV)
    keep = state.clone()
    o, snaps = gdn.decode_multi(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), state)
    torch.cuda.synchronize()
    assert torch.equal(state, keep)  # the state is only read
    o_ref, s_ref = oracle.decode_multi(*(to_f64(x[n]) for n in ("q", "k", "v", "g", "beta")), state0)
    og, sg = to_f64(o), to_f64(snaps)
    worst_o = max(rel(og[n, :, h], o_ref[n, :, h]) for n in range(N) for h in range(hv))
    worst_s = max(rel(sg[n, j, h], s_ref[n, j, h]) for n in range(N) for j in range(K) for h in range(hv))
    assert worst_o <= BAR[dtype] and worst_s <= BAR[dtype], (worst_o, worst_s)


def test_decode_multi_raw_inputs():
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    from test_gpu_input_side import raw_inputs
    N, K, hk, hv, d = 5, 4, 2, 4, 128
    x = raw_inputs(210, B=N, T=K, hk=hk, hv=hv, d=d, dtype="bf16")
    state0 = I.normal(211, "mtp_s0", (N, hv, d, d), std=0.05)
    o, snaps = gdn.decode_multi(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")),
                                torch.from_numpy(state0).float().to(DEV), qk_l2norm=True, gate_logits=True)
    torch.cuda.synchronize()
    q, k, g, b = oracle.prepare_inputs(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["g"]), to_f64(x["beta"]),
                                       qk_l2norm=True, gate_logits=True)
    o_ref, s_ref = oracle.decode_multi(q, k, to_f64(x["v"]), g, b, state0)
    og, sg = to_f64(o), to_f64(snaps)
    worst = max(rel(og[n, :, h], o_ref[n, :, h]) for n in range(N) for h in range(hv))
    worst_s = max(rel(sg[n, -1, h], s_ref[n, -1, h]) for n in range(N) for h in range(hv))
    assert worst <= BAR["bf16"] and worst_s <= BAR["bf16"], (worst, worst_s)


def test_decode_multi_equals_sequential_decode_steps():
    """K tokens in one pass against K single-token decode steps on the GPU
    (the same per-row arithmetic, so equal up to fp32 rounding)."""
    from linear_attention_sequence_sm_b200 import gdn
    N, K, hk, hv, d = 8, 5, 2, 4, 128
    x = {k_: v_.to(DEV) for k_, v_ in mtp_inputs(220, N, K, hk, hv, d, "bf16").items() if v_ is not None}
    state = torch.from_numpy(I.normal(221, "mtp_s0", (N, hv, d, d), std=0.05)).float().to(DEV)
    o, snaps = gdn.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
    seq = state.clone()
    for j in range(K):
        oj = gdn.decode_step(x["q"][:, j].contiguous(), x["k"][:, j].contiguous(), x["v"][:, j].contiguous(),
                             x["g"][:, j].contiguous(), x["beta"][:, j].contiguous(), seq)
        assert (oj.float() - o[:, j].float()).abs().max().item() < 2e-2
        assert torch.allclose(seq, snaps[:, j], rtol=1e-5, atol=1e-6)
    torch.cuda.synchronize()


def test_decode_commit():
    """Accepted prefixes 0..K and an out-of-range value: the state takes the
    snapshot of the accepted prefix, keeps itself for 0, is left alone (and
    counted) for a bad value."""
    from linear_attention_sequence_sm_b200 import gdn
    N, K, hk, hv, d = 6, 4, 1, 2, 128
    x = {k_: v_.to(DEV) for k_, v_ in mtp_inputs(230, N, K, hk, hv, d, "bf16").items() if v_ is not None}
    state = torch.from_numpy(I.normal(231, "mtp_s0", (N, hv, d, d), std=0.05)).float().to(DEV)
    before = state.clone()
    _, snaps = gdn.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
    accepted = torch.tensor([0, 1, 2, 3, 4, 7], dtype=torch.int32, device=DEV)
    bad = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn.decode_commit(snaps, accepted, state, bad_count=bad)
    torch.cuda.synchronize()
    for n, a in enumerate(accepted.tolist()):
        want = before[n] if a == 0 or a > K else snaps[n, a - 1]
        assert torch.equal(state[n], want), n
    assert bad.item() == 1


def test_draft_verify_loop_matches_recurrence():
    """Draft, verify, commit, repeat: the committed state equals the oracle's
    recurrence over the accepted tokens only."""
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    N, K, hk, hv, d = 4, 3, 2, 4, 128
    state0 = I.normal(240, "mtp_s0", (N, hv, d, d), std=0.05)
    state = torch.from_numpy(state0).float().to(DEV)
    ref = state0.copy()
    rng = np.random.default_rng(241)
    for it in range(4):
        x = mtp_inputs(242 + it, N, K, hk, hv, d, "f32")
        _, snaps = gdn.decode_multi(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), state)
        acc = rng.integers(0, K + 1, size=N).astype(np.int32)
        gdn.decode_commit(snaps, torch.from_numpy(acc).to(DEV), state)
        for n in range(N):
            for j in range(acc[n]):
                sl = lambda t: to_f64(t[n:n + 1, j])
                _, s1 = oracle.decode_step(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["g"]), sl(x["beta"]),
                                           ref[n:n + 1])
                ref[n] = s1[0]
    torch.cuda.synchronize()
    sg = to_f64(state)
    worst = max(rel(sg[n, h], ref[n, h]) for n in range(N) for h in range(hv))
    assert worst <= BAR["f32"], worst
