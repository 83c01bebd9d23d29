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


def gpu_prefill(inp, chunk, force_simt=False, final_state=True, initial_state="inp", split=False):
    from linear_attention_sequence_sm_b200 import gdn
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    s0 = d["initial_state"] if initial_state == "inp" else initial_state
    o, sf = gdn.chunk_forward(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=s0,
                              cu_seqlens=d["cu_seqlens"], chunk_size=chunk, output_final_state=final_state,
                              force_simt=force_simt, split=split)
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


def _seq_bounds(inp):
    """(start, end) token bounds of every sequence in the flattened token axis."""
    q = inp["q"]
    if inp["cu_seqlens"] is None:
        B, T = q.shape[0], q.shape[1]
        return [(b * T, (b + 1) * T) for b in range(B)]
    cu = inp["cu_seqlens"].tolist()
    return [(cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def _segment_rel(err2, ref2, starts):
    """Max over token segments (each from one start to the next) of
    sqrt(sum err2) / max(sqrt(sum ref2), 1e-30), per head column."""
    if len(starts) == 0:
        return 0.0
    e = np.add.reduceat(err2, starts, axis=0)
    r = np.add.reduceat(ref2, starts, axis=0)
    return float((np.sqrt(e) / np.maximum(np.sqrt(r), 1e-30)).max())


def full_prefill_errors(inp, o_gpu, sf_gpu, chunk=64, threads=None, kda=False):
    """Every (sequence, value head) unit of a prefill against the fp64 oracle.

    The oracle runs a few q/k heads at a time (with their value heads), so
    host memory stays bounded at full sizes.  Returns a dict:
      o_slice  max rel-L2 over (sequence, head) slices of o (the parity metric)
      o_chunk  max rel-L2 over (sequence, head, chunk of ``chunk`` tokens)
               slices of o, so that one wrong chunk cannot hide in a long slice
      state    max rel-L2 over the (sequence, head) final states
      units    (sequence, head) units compared
    With ``kda`` the gates are per key channel ([..., Hv, d_k]) and the
    oracle's KDA recurrence is the reference.
    """
    from oracle import oracle
    threads = threads or oracle.default_threads()
    hk, hv = inp["q"].shape[-2], inp["v"].shape[-2]
    G = hv // hk
    bounds = _seq_bounds(inp)
    N = len(bounds)
    seq_starts = np.array([a for a, b in bounds if b > a], dtype=np.int64)
    chunk_starts = np.array([t for a, b in bounds for t in range(a, b, chunk)], dtype=np.int64)
    dv = inp["v"].shape[-1]
    og_all = o_gpu.detach().reshape(-1, hv, dv)
    sg_all = None if sf_gpu is None else sf_gpu.detach()
    per_call = max(1, min(hk, -(-threads // max(1, N * G))))
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype(np.int64)
    res = {"o_slice": 0.0, "o_chunk": 0.0, "state": 0.0, "units": 0}
    for q0 in range(0, hk, per_call):
        q1 = min(hk, q0 + per_call)
        h0, h1 = q0 * G, q1 * G
        q = to_f64(inp["q"][..., q0:q1, :])
        k = to_f64(inp["k"][..., q0:q1, :])
        v = to_f64(inp["v"][..., h0:h1, :])
        g = to_f64(inp["g"][..., h0:h1, :]) if kda else to_f64(inp["g"][..., h0:h1])
        b = to_f64(inp["beta"][..., h0:h1])
        s0 = None if inp["initial_state"] is None else to_f64(inp["initial_state"][:, h0:h1])
        run = oracle.kda_recurrent if kda else oracle.recurrent
        o_ref, s_ref = run(q, k, v, g, b, initial_state=s0, cu_seqlens=cu, threads=threads)
        o_ref = np.asarray(o_ref).reshape(-1, h1 - h0, dv)
        og = to_f64(og_all[:, h0:h1].cpu())
        err2 = ((og - o_ref) ** 2).sum(axis=-1)
        ref2 = (o_ref ** 2).sum(axis=-1)
        res["o_slice"] = max(res["o_slice"], _segment_rel(err2, ref2, seq_starts))
        res["o_chunk"] = max(res["o_chunk"], _segment_rel(err2, ref2, chunk_starts))
        if sg_all is not None:
            sg = to_f64(sg_all[:, h0:h1].cpu())
            e = np.sqrt(((sg - s_ref) ** 2).sum(axis=(-2, -1)))
            r = np.maximum(np.sqrt((s_ref ** 2).sum(axis=(-2, -1))), 1e-30)
            res["state"] = max(res["state"], float((e / r).max()))
        res["units"] += N * (h1 - h0)
        del q, k, v, g, b, s0, o_ref, s_ref, og, err2, ref2
    return res
