"""Seeded synthetic inputs for the gated delta rule workloads.

This module is shared by the tests, the benchmark and the smoke check.  It
holds none of the method's arithmetic: it draws random numbers, applies the
input recipe (L2-normalised q/k, sigmoid beta, softplus-shaped log-decay g),
and rounds to the storage dtype.  Both the CUDA path and the fp64 oracle
receive exactly the arrays produced here.

Random numbers: a counter-based splitmix64 stream (Steele, Lea and Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014) turned into
uniforms with 53-bit mantissas and into normals with the Box-Muller
transform.  Every tensor gets its own stream derived from (seed, tag), so a
tensor's values do not depend on which other tensors were drawn.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, tag: str) -> np.uint64:
    h = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    for ch in tag.encode():
        h = _mix(h ^ np.uint64(ch) + _GOLDEN)
    return h[0]


def uniform(seed: int, tag: str, n: int, offset: int = 0) -> np.ndarray:
    """n uniforms in (0, 1), element i from counter offset + i of stream (seed, tag)."""
    key = _stream_key(seed, tag)
    with np.errstate(over="ignore"):
        ctr = np.arange(offset + 1, offset + n + 1, dtype=np.uint64) * _GOLDEN + key
        bits = _mix(ctr)
    return ((bits >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(seed: int, tag: str, shape, mean: float = 0.0, std: float = 1.0, offset: int = 0) -> np.ndarray:
    """Box-Muller normals (fp64) of the given shape from stream (seed, tag).

    Element i of the stream uses uniforms 2*(i//2) and 2*(i//2)+1, so a slab
    that starts at an even ``offset`` reproduces the same values as drawing
    the whole stream at once.
    """
    if offset % 2:
        raise ValueError("slab offset must be even")
    n = int(np.prod(shape))
    m = (n + 1) // 2
    u = uniform(seed, tag, 2 * m, offset)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    th = 2.0 * math.pi * u[1::2]
    z = np.empty(2 * m)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return (mean + std * z[:n]).reshape(shape)


def _slabbed(seed: int, tag: str, shape, fn, out_dtype, row_elems: int, slab_rows: int = 8192):
    """Draw normals for ``shape`` slab by slab along the leading flattened rows
    (each row = ``row_elems`` elements), apply ``fn`` (elementwise or per-row)
    and store into a torch tensor of ``out_dtype``.  Slabs are drawn on a pool
    of host threads (numpy releases the interpreter lock inside its array
    operations); every slab is a fixed range of counters of the stream, so the
    values do not depend on the thread count or the order of completion."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    import torch
    n = int(np.prod(shape))
    rows = n // row_elems
    out = torch.empty(n, dtype=out_dtype)

    def slab(r0):
        r1 = min(rows, r0 + slab_rows)
        off = r0 * row_elems
        z = normal(seed, tag, ((r1 - r0), row_elems), offset=off)
        out[off:r1 * row_elems] = torch.from_numpy(np.ascontiguousarray(fn(z).reshape(-1))).to(out_dtype)

    starts = list(range(0, rows, slab_rows))
    workers = min(len(starts), len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else 8, 32)
    if workers <= 1:
        for r0 in starts:
            slab(r0)
    else:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(slab, starts))
    return out.reshape(shape)


def randint(seed: int, tag: str, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers uniform in [lo, hi] (inclusive)."""
    u = uniform(seed, tag, n)
    return np.minimum(lo + np.floor(u * (hi - lo + 1)).astype(np.int64), hi)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def l2_normalise(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


@dataclass
class Workload:
    """One gated-delta-rule problem: shapes plus the recipe of its values."""
    name: str
    batch: int                 # B (1 for packed varlen)
    seq_len: int               # T per batch row (total tokens for packed varlen)
    hk: int
    hv: int
    d: int
    chunk: int
    dtype: str                 # "f32" or "bf16": storage type of q, k, v, o
    g_shift: float = 0.0       # g = -g_scale * softplus(N(0,1) + g_shift)
    g_scale: float = 1.0
    s0_std: float = 0.0        # 0: zero initial state
    seq_lens: list | None = None   # packed varlen lengths (then batch == 1)
    seed: int = 1000
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens) if self.seq_lens is not None else self.batch

    @property
    def total_tokens(self) -> int:
        return self.batch * self.seq_len

    def cu_seqlens(self) -> np.ndarray | None:
        if self.seq_lens is None:
            return None
        return np.concatenate([[0], np.cumsum(self.seq_lens)]).astype(np.int32)


def tiny_fp32(seed: int = 1001) -> Workload:
    return Workload("tiny_fp32_B1_T64_h2x2_d16_C16", 1, 64, 2, 2, 16, 16, "f32", seed=seed)


def prefill_bf16(seed: int = 1002) -> Workload:
    return Workload("prefill_bf16_B4_T4096_hk16_hv32_d128_C64", 4, 4096, 16, 32, 128, 64, "bf16",
                    g_shift=2.0, g_scale=0.1, seed=seed)


def long_bf16(seed: int = 1003) -> Workload:
    return Workload("long_bf16_B1_T65536_hk16_hv48_d128_C64", 1, 65536, 16, 48, 128, 64, "bf16",
                    s0_std=0.02, seed=seed)


def varlen_bf16(seed: int = 1005) -> Workload:
    lens = randint(seed, "seq_lens", 32, 128, 8192).tolist()
    return Workload("varlen_bf16_N32_L128-8192_hk16_hv32_d128_C64", 1, int(sum(lens)), 16, 32, 128, 64,
                    "bf16", s0_std=0.02, seq_lens=lens, seed=seed)


@dataclass
class DecodeWorkload:
    name: str
    num_seqs: int
    hk: int
    hv: int
    d: int
    dtype: str
    steps: int
    s0_std: float
    seed: int = 1004


def decode_bf16(seed: int = 1004) -> DecodeWorkload:
    return DecodeWorkload("decode_bf16_N256_hk16_hv32_d128", 256, 16, 32, 128, "bf16", 512, 0.05, seed)


def _round(x: np.ndarray, dtype: str):
    """Round an fp64 array to the storage dtype; returns a torch CPU tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.float32) if dtype == "f32" else t.to(torch.bfloat16)


def _torch_dtype(dtype: str):
    import torch
    return torch.float32 if dtype == "f32" else torch.bfloat16


def make_prefill_inputs(w: Workload):
    """Draw q, k, v, g, beta, initial_state, cu_seqlens for workload ``w``.

    Returns a dict of torch CPU tensors: q, k [B,T,Hk,d]; v [B,T,Hv,d] in the
    storage dtype; g, beta [B,T,Hv] fp32; initial_state [N,Hv,d,d] fp32 or
    None; cu_seqlens int32 [N+1] or None.  Values are drawn in fp64 (q and k
    L2-normalised per token and head in fp64) and rounded once to the
    storage dtype (round-to-nearest-even).
    """
    import torch
    B, T, hk, hv, d = w.batch, w.seq_len, w.hk, w.hv, w.d
    s = w.seed
    st = _torch_dtype(w.dtype)
    ident = lambda z: z
    out = {
        "q": _slabbed(s, "q", (B, T, hk, d), l2_normalise, st, d),
        "k": _slabbed(s, "k", (B, T, hk, d), l2_normalise, st, d),
        "v": _slabbed(s, "v", (B, T, hv, d), ident, st, d),
        "g": _slabbed(s, "g", (B, T, hv), lambda z: -w.g_scale * _softplus(z + w.g_shift), torch.float32, hv),
        "beta": _slabbed(s, "beta", (B, T, hv), _sigmoid, torch.float32, hv),
        "initial_state": None, "cu_seqlens": None,
    }
    if w.s0_std > 0:
        out["initial_state"] = _slabbed(s, "s0", (w.num_seqs, hv, d, d), lambda z: w.s0_std * z,
                                        torch.float32, d)
    cu = w.cu_seqlens()
    if cu is not None:
        out["cu_seqlens"] = torch.from_numpy(cu)
    return out


def make_raw_prefill_inputs(w: Workload):
    """The workload's shapes with raw projections, for the input side done in
    the kernels (GDN_FLAG_QK_L2NORM, GDN_FLAG_GATE_LOGITS): q and k rows
    N(0,1) times a per-(token, head) norm factor uniform in [0.3, 6] (not
    normalised), v N(0,1), decay logits a ~ N(1.5, 1) (alpha = sigmoid(a)) and
    write logits b ~ N(0, 1) (beta = sigmoid(b)); states and cu_seqlens as in
    make_prefill_inputs."""
    import torch
    base = make_prefill_inputs(w)
    B, T, hk, hv, d = w.batch, w.seq_len, w.hk, w.hv, w.d
    s = w.seed
    st = _torch_dtype(w.dtype)
    rows = B * T * hk

    def raw(tag):
        def f(z):
            return z
        x = _slabbed(s, tag, (B, T, hk, d), f, torch.float32, d)
        sc = torch.from_numpy(0.3 + 5.7 * uniform(s, tag + "_scale", rows)).float().reshape(B, T, hk, 1)
        return (x * sc).to(st)

    base["q"], base["k"] = raw("raw_q"), raw("raw_k")
    base["g"] = _slabbed(s, "raw_a", (B, T, hv), lambda z: z + 1.5, torch.float32, hv)
    base["beta"] = _slabbed(s, "raw_b", (B, T, hv), lambda z: z, torch.float32, hv)
    return base


def make_kda_gates(w: Workload):
    """Kimi Delta Attention's per-key-channel log-decay, [B, T, Hv, d] fp32,
    with the scalar gate's recipe drawn once per channel:
    g = -g_scale * softplus(N(0,1) + g_shift)."""
    import torch
    B, T, hv, d = w.batch, w.seq_len, w.hv, w.d
    return _slabbed(w.seed, "kda_g", (B, T, hv, d), lambda z: -w.g_scale * _softplus(z + w.g_shift),
                    torch.float32, d)


def make_output_gate(w: Workload):
    """The output side's gate pre-activation z, shaped like o: N(0, 2^2)
    (SiLU then spans its negative dip and its near-identity range), rounded
    once to the storage dtype."""
    import torch
    B, T, hv, d = w.batch, w.seq_len, w.hv, w.d
    return _slabbed(w.seed, "out_gate", (B, T, hv, d), lambda z: 2.0 * z, _torch_dtype(w.dtype), d)


def make_output_weight(w: Workload):
    """The output side's per-channel scale, shared by the value heads:
    N(1, 0.1^2) fp32 (a trained RMSNorm scale stays near 1)."""
    import torch
    return torch.from_numpy(normal(w.seed, "out_weight", (w.d,), mean=1.0, std=0.1)).to(torch.float32)


def make_decode_inputs(w: DecodeWorkload, step: int):
    """Fresh per-step q, k [N,Hk,d], v [N,Hv,d], g, beta [N,Hv] (seed + step)."""
    import torch
    s = w.seed + step
    N, hk, hv, d = w.num_seqs, w.hk, w.hv, w.d
    q = l2_normalise(normal(s, "dq", (N, hk, d)))
    k = l2_normalise(normal(s, "dk", (N, hk, d)))
    v = normal(s, "dv", (N, hv, d))
    beta = _sigmoid(normal(s, "dbeta", (N, hv)))
    g = -_softplus(normal(s, "dg", (N, hv)))
    return {"q": _round(q, w.dtype), "k": _round(k, w.dtype), "v": _round(v, w.dtype),
            "g": torch.from_numpy(g).to(torch.float32), "beta": torch.from_numpy(beta).to(torch.float32)}


def make_kda_decode_gates(w: DecodeWorkload, step: int):
    """Kimi Delta Attention decode: a per-key-channel log-decay [N, Hv, d],
    -softplus(N(0,1)) per channel (seed + step)."""
    import torch
    g = -_softplus(normal(w.seed + step, "dkda_g", (w.num_seqs, w.hv, w.d)))
    return torch.from_numpy(g).to(torch.float32)


def make_decode_state(w: DecodeWorkload):
    import torch
    return torch.from_numpy(normal(w.seed, "state", (w.num_seqs, w.hv, w.d, w.d), std=w.s0_std)).to(
        torch.float32)


def custom(name: str, batch: int, seq_len: int, hk: int, hv: int, d: int, chunk: int, dtype: str,
           seed: int, g_shift: float = 0.0, g_scale: float = 1.0, s0_std: float = 0.0,
           seq_lens: list | None = None) -> Workload:
    """A workload with the same value recipe at other sizes (parity cases)."""
    if seq_lens is not None:
        batch, seq_len = 1, int(sum(seq_lens))
    return Workload(name, batch, seq_len, hk, hv, d, chunk, dtype, g_shift, g_scale, s0_std,
                    list(seq_lens) if seq_lens is not None else None, seed)
