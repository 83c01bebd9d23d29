"""GPU parity of the decode step (gdn_decode_step) against the fp64 oracle,
through the C ABI; the state carries across steps in place."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, to_f64

pytestmark = pytest.mark.gpu


def _rel(x, ref, axes):
    """Per-(sequence, head) relative L2 errors, norms over ``axes``."""
    e = np.sqrt(((x - ref) ** 2).sum(axis=axes))
    return e / np.maximum(np.sqrt((ref ** 2).sum(axis=axes)), 1e-30)


def _run(w, steps):
    """``steps`` decode steps of workload ``w`` on the GPU (state in place) and
    in the oracle; every (sequence, head) unit's output compared at every
    step, and the state after the last step.  Returns (worst o, worst state)."""
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    dev = torch.device("cuda:0")
    state = I.make_decode_state(w)
    ref_state = to_f64(state)
    st = state.to(dev)
    worst_o = 0.0
    for step in range(steps):
        x = I.make_decode_inputs(w, step)
        d = {k: v.to(dev) for k, v in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], st)
        torch.cuda.synchronize()
        xs = {k: to_f64(v) for k, v in x.items()}
        o_ref, ref_state = oracle.decode_step(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], ref_state)
        worst_o = max(worst_o, float(_rel(to_f64(o), o_ref, (-1,)).max()))
    worst_s = float(_rel(to_f64(st), ref_state, (-2, -1)).max())
    return worst_o, worst_s


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 16, 64])
def test_decode_small(dtype, d):
    w = I.DecodeWorkload(f"decode_{dtype}_{d}", 6, 2, 4, d, dtype, 20, 0.05, seed=41 + d)
    eo, es = _run(w, w.steps)
    assert eo <= BAR[dtype] and es <= BAR[dtype], (eo, es)


def test_decode_full_size_all_units():
    """256 sequences, 16/32 heads, d=128, fp32 state of 512 MiB updated in
    place; every (sequence, head) unit checked at each of 64 steps, and the
    whole state after them."""
    w = I.decode_bf16()
    eo, es = _run(w, 64)
    print(f"PARITY {w.name}: 64 steps, all {w.num_seqs * w.hv} units: o {eo:.3e} state {es:.3e}")
    assert eo <= BAR["bf16"] and es <= BAR["bf16"], (eo, es)


def test_decode_dv_not_multiple_of_batch():
    """d_v = 40 (not a multiple of the row batch) with d_k = 128."""
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    rng = np.random.default_rng(3)
    N, hk, hv, dk, dv = 3, 1, 2, 128, 40
    q = rng.standard_normal((N, hk, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((N, hk, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, hv, dv))
    g = -np.logaddexp(0, rng.standard_normal((N, hv)))
    b = 1 / (1 + np.exp(-rng.standard_normal((N, hv))))
    S = 0.1 * rng.standard_normal((N, hv, dv, dk))
    dev = torch.device("cuda:0")
    t = lambda a: torch.tensor(a, dtype=torch.float32, device=dev)
    st = t(S)
    o = gdn.decode_step(t(q), t(k), t(v), t(g), t(b), st)
    o_ref, s_ref = oracle.decode_step(q, k, v, g, b, S)
    np.testing.assert_allclose(to_f64(o), o_ref, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(to_f64(st), s_ref, rtol=1e-4, atol=1e-5)
