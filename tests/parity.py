"""Helpers for GPU-vs-oracle parity: run the CUDA path through the C ABI,
run the fp64 oracle on the same seeded inputs, and compare per
(sequence, value head) slice with the max relative L2 error."""
from __future__ import annotations

import numpy as np
import torch

from conftest import rel_l2_per_slice  # noqa: F401  (re-export)

BAR = {"f32": 1e-4, "bf16": 2e-2}


def to_f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def gpu_prefill(inp, chunk, force_simt=False, final_state=True, initial_state="inp"):
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    s0 = d["initial_state"] if initial_state == "inp" else initial_state
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=s0,
                              cu_seqlens=d["cu_seqlens"], chunk_size=chunk, output_final_state=final_state,
                              force_simt=force_simt)
    torch.cuda.synchronize()
    return o, sf


def oracle_prefill(inp, units=None):
    from oracle import oracle
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    return oracle.recurrent(to_f64(inp["q"]), to_f64(inp["k"]), to_f64(inp["v"]), to_f64(inp["g"]),
                            to_f64(inp["beta"]), initial_state=to_f64(inp["initial_state"]), cu_seqlens=cu,
                            units=units)


def slices(inp):
    """(sequence, token slice) pairs of the packed/batched layout."""
    q = inp["q"]
    if inp["cu_seqlens"] is None:
        B, T = q.shape[0], q.shape[1]
        return [(b, b * T, (b + 1) * T) for b in range(B)]
    cu = inp["cu_seqlens"].tolist()
    return [(n, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def prefill_errors(inp, o_gpu, sf_gpu, o_ref, sf_ref, units=None):
    """Max rel-L2 over (sequence, head) slices of o and of the final state."""
    hv = inp["v"].shape[-2]
    dv = inp["v"].shape[-1]
    og = to_f64(o_gpu).reshape(-1, hv, dv)
    orf = np.asarray(o_ref).reshape(-1, hv, dv)
    sg = None if sf_gpu is None else to_f64(sf_gpu)
    worst_o = worst_s = 0.0
    for n, a, b in slices(inp):
        for h in range(hv):
            if units is not None and n * hv + h not in units:
                continue
            if b > a:
                ref = orf[a:b, h]
                err = np.linalg.norm(og[a:b, h] - ref) / max(np.linalg.norm(ref), 1e-30)
                worst_o = max(worst_o, err)
            if sg is not None:
                ref = sf_ref[n, h]
                err = np.linalg.norm(sg[n, h] - ref) / max(np.linalg.norm(ref), 1e-30)
                worst_s = max(worst_s, err)
    return worst_o, worst_s


def oracle_units_sliced(inp, units, hv, hk):
    """Oracle outputs for the listed (sequence, head) units, each run on its own
    head's slice of the inputs (keeps host memory bounded at full sizes).
    Returns {unit: (o [T_n, d_v], final state [d_v, d_k])}."""
    from oracle import oracle
    G = hv // hk
    q, k, v = inp["q"], inp["k"], inp["v"]
    res = {}
    for u in units:
        n, h = divmod(u, hv)
        hq = h // G
        if inp["cu_seqlens"] is None:
            qs, ks = q[n, :, hq:hq + 1], k[n, :, hq:hq + 1]
            vs, gs, bs = v[n, :, h:h + 1], inp["g"][n, :, h:h + 1], inp["beta"][n, :, h:h + 1]
        else:
            cu = inp["cu_seqlens"].tolist()
            a, b = cu[n], cu[n + 1]
            qs, ks = q[0, a:b, hq:hq + 1], k[0, a:b, hq:hq + 1]
            vs, gs, bs = v[0, a:b, h:h + 1], inp["g"][0, a:b, h:h + 1], inp["beta"][0, a:b, h:h + 1]
        s0 = None if inp["initial_state"] is None else to_f64(inp["initial_state"][n:n + 1, h:h + 1])
        o, sf = oracle.recurrent(to_f64(qs)[None], to_f64(ks)[None], to_f64(vs)[None], to_f64(gs)[None],
                                 to_f64(bs)[None], initial_state=s0)
        res[u] = (o[0, :, 0], sf[0, 0])
    return res
