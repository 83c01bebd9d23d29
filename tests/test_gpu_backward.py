"""GPU parity of the gradients (training) against the fp64 oracle's reverse
mode of the token recurrence ("Architecture Thread I", the Gated DeltaNet
section; "Gated Attention Architectures", sections 2 and 3), per
(sequence, head) slice: dq, dk per q/k head, dv, dg, dbeta per value head,
and the initial-state gradient.

Bars, GRAD_BAR by input type:
- fp32 inputs: the products run in fp32 on CUDA cores.  fp32 rounding over
  sums of O(C d) terms per chunk, carried through T / C chunks of the
  state-gradient recurrence, stays well below 1e-4 relative on these sizes;
  2e-4 leaves room for the atomic summation order of dq, dk, dg and dbeta.
- bf16 inputs: the products run on the tensor cores, each fp32 operand
  split into a bf16 value and a bf16 residual (three products per tile,
  about 16 mantissa bits, fp32 accumulation); the same 2e-4 holds."""
import numpy as np
import pytest
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import to_f64, slices

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GRAD_BAR = {"f32": 2e-4, "bf16": 2e-4}


def bwd_inputs(seed, B, T, hk, hv, d, dtype, seq_lens=None, s0_std=0.05):
    w = I.custom(f"bwd_{seed}", batch=B, seq_len=T, hk=hk, hv=hv, d=d, chunk=32, dtype=dtype, seed=seed,
                 s0_std=s0_std, seq_lens=seq_lens)
    inp = I.make_prefill_inputs(w)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    inp["dO"] = torch.from_numpy(I.normal(seed, "bwd_do", tuple(inp["v"].shape))).to(td)
    inp["dSf"] = torch.from_numpy(I.normal(seed, "bwd_dsf", (w.num_seqs, hv, d, d), std=0.1)).float()
    return inp


def run_both(inp, with_dsf=True):
    from linear_attention_sequence_sm_b200 import gdn
    from oracle import oracle
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    gg = gdn.chunk_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"],
                            d_final_state=d["dSf"] if with_dsf else None, initial_state=d["initial_state"],
                            cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    ref = oracle.backward(*(to_f64(inp[n]) for n in ("q", "k", "v", "g", "beta", "dO")),
                          dS_final=to_f64(inp["dSf"]) if with_dsf else None,
                          initial_state=to_f64(inp["initial_state"]), cu_seqlens=cu)
    return gg, ref


def worst_errors(inp, gg, ref):
    """Max rel-L2 over (sequence, head) slices of each gradient."""
    hk, hv = inp["q"].shape[-2], inp["v"].shape[-2]
    out = {}
    for name, heads in (("dq", hk), ("dk", hk), ("dv", hv), ("dg", hv), ("dbeta", hv)):
        got = to_f64(gg[name]).reshape(-1, heads, *gg[name].shape[len(inp["q"].shape[:-2]) + 1:])
        want = np.asarray(ref[name]).reshape(got.shape)
        w = 0.0
        for n, a, b in slices(inp):
            for h in range(heads):
                if b > a:
                    r = want[a:b, h]
                    w = max(w, np.linalg.norm(got[a:b, h] - r) / max(np.linalg.norm(r), 1e-30))
        out[name] = w
    g0, r0 = to_f64(gg["d_initial_state"]), ref["dS0"]
    out["dS0"] = max(np.linalg.norm(g0[n, h] - r0[n, h]) / max(np.linalg.norm(r0[n, h]), 1e-30)
                     for n in range(r0.shape[0]) for h in range(hv))
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [128, 64])
def test_backward_parity(dtype, d):
    inp = bwd_inputs(300 + d, B=2, T=100, hk=2, hv=4, d=d, dtype=dtype)
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(dtype, d, errs)
    assert max(errs.values()) <= GRAD_BAR[dtype], errs


def test_backward_varlen_edges():
    lens = [1, 31, 32, 33, 0, 70, 5]
    inp = bwd_inputs(310, B=1, T=sum(lens), hk=1, hv=2, d=128, dtype="bf16", seq_lens=lens)
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs
    # the empty sequence passes its final-state gradient straight through
    assert torch.allclose(gg["d_initial_state"][4], inp["dSf"][4].to(DEV), rtol=0, atol=0)


def test_backward_small_dims_without_final_gradient():
    inp = bwd_inputs(320, B=3, T=45, hk=1, hv=3, d=16, dtype="f32")
    gg, ref = run_both(inp, with_dsf=False)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["f32"], errs


# ---- the tensor-core form (bf16, d = 128: factors, state chains, gradients over chunks of 64)

def test_backward_tc_chunk_boundaries():
    """Sequences on both sides of the 64-token chunks the tensor-core form
    uses (one, two and three chunks, a full and a one-token last chunk)."""
    lens = [63, 64, 65, 127, 128, 129, 1, 192]
    inp = bwd_inputs(330, B=1, T=sum(lens), hk=2, hv=4, d=128, dtype="bf16", seq_lens=lens)
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs


def test_backward_tc_long_chains():
    """2048 tokens: the state and state-gradient chains over 32 chunks."""
    inp = bwd_inputs(331, B=1, T=2048, hk=1, hv=2, d=128, dtype="bf16")
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs


def test_backward_tc_strong_decay():
    """Gates at and just above the kernels' floor (-20): the decays
    gamma_r = e^(G_r) underflow to zero inside every chunk (the oracle reads
    g unfloored, so gates below the floor are left to the next test)."""
    inp = bwd_inputs(332, B=2, T=150, hk=1, hv=2, d=128, dtype="bf16")
    g = inp["g"].clone()
    g[:, ::3] = -19.5
    g[:, 1::3] = -20.0
    inp["g"] = g
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs


@pytest.mark.parametrize("force_simt", [False, True])
def test_backward_dg_zero_below_floor(force_simt):
    """The kernels read g as max(g, -20), whose derivative is zero below the
    floor: dg is exactly zero there, and the other gradients match the same
    inputs with those gates raised to the floor."""
    from linear_attention_sequence_sm_b200 import gdn
    inp = bwd_inputs(334, B=2, T=150, hk=1, hv=2, d=128, dtype="bf16")
    g = inp["g"].clone()
    g[:, 5::7] = -25.0
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    below = g.to(DEV) < -20
    a = gdn.chunk_backward(d["q"], d["k"], d["v"], g.to(DEV), d["beta"], d["dO"], d_final_state=d["dSf"],
                           initial_state=d["initial_state"], force_simt=force_simt)
    b = gdn.chunk_backward(d["q"], d["k"], d["v"], g.clamp_min(-20).to(DEV), d["beta"], d["dO"],
                           d_final_state=d["dSf"], initial_state=d["initial_state"], force_simt=force_simt)
    assert torch.count_nonzero(a["dg"][below]) == 0
    assert torch.allclose(a["dg"][~below], b["dg"][~below], rtol=1e-5, atol=1e-6)
    for name in ("dq", "dk", "dv", "dbeta", "d_initial_state"):
        assert torch.allclose(a[name], b[name], rtol=1e-5, atol=1e-6), name


def test_backward_tc_matches_single_kernel():
    """The tensor-core form and the single-kernel form (GDN_FLAG_FORCE_SIMT)
    agree on a ragged batch, with and without an initial state."""
    from linear_attention_sequence_sm_b200 import gdn
    for s0 in (0.05, 0.0):
        inp = bwd_inputs(333, B=3, T=200, hk=2, hv=4, d=128, dtype="bf16", s0_std=s0)
        d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
        args = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"])
        kw = dict(d_final_state=d["dSf"], initial_state=d["initial_state"])
        a = gdn.chunk_backward(*args, **kw)
        b = gdn.chunk_backward(*args, force_simt=True, **kw)
        for name in ("dq", "dk", "dv", "dg", "dbeta", "d_initial_state"):
            x, y = a[name].double(), b[name].double()
            rel = ((x - y).norm() / y.norm().clamp_min(1e-30)).item()
            assert rel <= 2 * GRAD_BAR["bf16"], (s0, name, rel)


@pytest.mark.parametrize("case", ["bench_4x4096", "long_65536"])
def test_backward_tc_full_size(case):
    """Full size: the tensor-core form against the single-kernel form (itself
    checked against the oracle above) on the 4 x 4096 bench workload (16 q/k,
    32 value heads: every item and unit) and on one 65,536-token sequence
    (chains of 1024 chunks), per (sequence, head) slice of every gradient."""
    from linear_attention_sequence_sm_b200 import gdn
    if case == "bench_4x4096":
        w = I.custom("bwd_full", batch=4, seq_len=4096, hk=16, hv=32, d=128, chunk=64, dtype="bf16", seed=41,
                     s0_std=0.05)
    else:
        w = I.custom("bwd_long", batch=1, seq_len=65536, hk=2, hv=4, d=128, chunk=64, dtype="bf16", seed=42,
                     s0_std=0.05)
    inp = I.make_prefill_inputs(w)
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    dO = torch.from_numpy(I.normal(w.seed, "bwd_do", tuple(inp["v"].shape))).to(torch.bfloat16).to(DEV)
    dSf = torch.from_numpy(I.normal(w.seed, "bwd_dsf", (w.num_seqs, w.hv, 128, 128), std=0.1)).float().to(DEV)
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"], dO)
    a = gdn.chunk_backward(*args, d_final_state=dSf, initial_state=d["initial_state"])
    b = gdn.chunk_backward(*args, d_final_state=dSf, initial_state=d["initial_state"], force_simt=True)
    torch.cuda.synchronize()
    worst = {}
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        x, y = a[name].double(), b[name].double()
        heads = x.shape[2]
        x = x.reshape(w.batch, w.seq_len, heads, -1)
        y = y.reshape(w.batch, w.seq_len, heads, -1)
        diff = (x - y).norm(dim=(1, 3)) / y.norm(dim=(1, 3)).clamp_min(1e-30)  # per (sequence, head)
        worst[name] = diff.max().item()
    x, y = a["d_initial_state"].double(), b["d_initial_state"].double()
    worst["dS0"] = ((x - y).norm(dim=(2, 3)) / y.norm(dim=(2, 3)).clamp_min(1e-30)).max().item()
    print(case, worst)
    assert max(worst.values()) <= 2 * GRAD_BAR["bf16"], worst


@pytest.mark.parametrize("hk,hv", [(2, 2), (1, 3), (2, 6)])
def test_backward_tc_head_groups(hk, hv):
    """One, three and three value heads per q/k head: the gradient kernel
    takes 2 x (Hv / Hk) units per (chunk, q/k head) and sums their dq and dk
    in registers; the T tiles are loaded once per value head."""
    inp = bwd_inputs(335 + hv, B=2, T=130, hk=hk, hv=hv, d=128, dtype="bf16")
    gg, ref = run_both(inp)
    errs = worst_errors(inp, gg, ref)
    print(hk, hv, errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs


def test_backward_tc_optional_arguments():
    """The tensor-core form without a final-state gradient (zeros) and with
    and without the initial-state gradient output."""
    from linear_attention_sequence_sm_b200 import gdn
    inp = bwd_inputs(340, B=2, T=150, hk=1, hv=2, d=128, dtype="bf16")
    gg, ref = run_both(inp, with_dsf=False)
    errs = worst_errors(inp, gg, ref)
    print(errs)
    assert max(errs.values()) <= GRAD_BAR["bf16"], errs
    d = {k: (v.to(DEV) if v is not None else None) for k, v in inp.items()}
    nd = gdn.chunk_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], initial_state=d["initial_state"],
                            want_d_initial_state=False)
    assert nd["d_initial_state"] is None
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        assert torch.allclose(nd[name], gg[name], rtol=1e-5, atol=1e-6), name
