"""GPU parity of the decode step (gdn_decode_step) against the fp64 oracle,
through the C ABI; the state carries across steps in place."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import BAR, to_f64

pytestmark = pytest.mark.gpu


def _run(w, steps, units=None, dtype="bf16"):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    dev = torch.device("cuda:0")
    state = I.make_decode_state(w)
    ref_state = to_f64(state)
    if units is not None:
        ref_state = ref_state.copy()
    st = state.to(dev)
    worst_o = 0.0
    for step in range(steps):
        x = I.make_decode_inputs(w, step)
        d = {k: v.to(dev) for k, v in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], st)
        torch.cuda.synchronize()
        xs = {k: to_f64(v) for k, v in x.items()}
        if units is None:
            o_ref, ref_state = oracle.decode_step(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], ref_state)
            og = to_f64(o)
            for n in range(w.num_seqs):
                for h in range(w.hv):
                    e = np.linalg.norm(og[n, h] - o_ref[n, h]) / max(np.linalg.norm(o_ref[n, h]), 1e-30)
                    worst_o = max(worst_o, e)
        else:
            # sampled units: run the oracle on those (sequence, head) pairs only
            og = to_f64(o)
            for u in units:
                n, h = divmod(u, w.hv)
                hq = h // (w.hv // w.hk)
                o_ref, s_new = oracle.decode_step(xs["q"][n:n + 1, hq:hq + 1], xs["k"][n:n + 1, hq:hq + 1],
                                                  xs["v"][n:n + 1, h:h + 1], xs["g"][n:n + 1, h:h + 1],
                                                  xs["beta"][n:n + 1, h:h + 1], ref_state[n:n + 1, h:h + 1])
                ref_state[n, h] = s_new[0, 0]
                e = np.linalg.norm(og[n, h] - o_ref[0, 0]) / max(np.linalg.norm(o_ref[0, 0]), 1e-30)
                worst_o = max(worst_o, e)
    sg = to_f64(st)
    worst_s = 0.0
    for n in range(w.num_seqs):
        for h in range(w.hv):
            if units is not None and n * w.hv + h not in units:
                continue
            e = np.linalg.norm(sg[n, h] - ref_state[n, h]) / max(np.linalg.norm(ref_state[n, h]), 1e-30)
            worst_s = max(worst_s, e)
    return worst_o, worst_s


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 16, 64])
def test_decode_small(dtype, d):
    w = I.DecodeWorkload(f"decode_{dtype}_{d}", 6, 2, 4, d, dtype, 20, 0.05, seed=41 + d)
    eo, es = _run(w, w.steps)
    assert eo <= BAR[dtype] and es <= BAR[dtype], (eo, es)


def test_decode_full_size_sampled():
    """256 sequences, 16/32 heads, d=128, fp32 state of 512 MiB updated in
    place; 24 steps checked on 6 sampled (sequence, head) units."""
    w = I.decode_bf16()
    units = [0, 31, 4000, 5555, 8000, 256 * 32 - 1]
    eo, es = _run(w, 24, units=units)
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
