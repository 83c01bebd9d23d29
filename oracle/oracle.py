"""ctypes front end of the fp64 CPU oracle for the gated delta rule.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the product path
(``linear_attention_sequence_sm_b200``) never does.  The arithmetic lives in
``gdn_oracle.c``; this file only builds that file with gcc, marshals numpy
arrays, and hands back numpy arrays.

Readings of the pages (see ``gdn_oracle.c`` for the formulas):
state S is d_v x d_k, o_t = S_t q_t after the update at t, alpha = exp(g),
g and beta per token per value head, value head h reads q/k head
h // (Hv // Hk), NULL initial state = zeros.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle (plain C11, fp64, no fast-math) into a shared library.
    A library is reused only if it was built from a source of the same
    content (its SHA-256 is kept beside it), whatever the files' times."""
    import hashlib
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    stamp = out + ".sha256"
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    return out


class _Problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int64),
        ("cu_seqlens", ctypes.POINTER(ctypes.c_int64)),
        ("hk", ctypes.c_int32), ("hv", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
        ("q", ctypes.POINTER(ctypes.c_double)), ("k", ctypes.POINTER(ctypes.c_double)),
        ("v", ctypes.POINTER(ctypes.c_double)), ("g", ctypes.POINTER(ctypes.c_double)),
        ("beta", ctypes.POINTER(ctypes.c_double)),
        ("s0", ctypes.POINTER(ctypes.c_double)),
        ("o", ctypes.POINTER(ctypes.c_double)),
        ("s_final", ctypes.POINTER(ctypes.c_double)),
    ]


class _ChunkOut(ctypes.Structure):
    _fields_ = [
        ("chunk", ctypes.c_int32),
        ("gcum", ctypes.POINTER(ctypes.c_double)), ("tmat", ctypes.POINTER(ctypes.c_double)),
        ("w", ctypes.POINTER(ctypes.c_double)), ("ut", ctypes.POINTER(ctypes.c_double)),
        ("u", ctypes.POINTER(ctypes.c_double)), ("sc", ctypes.POINTER(ctypes.c_double)),
    ]


class _Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.POINTER(ctypes.c_double)) for n in ("dO", "dSf", "dq", "dk", "dv", "dg", "dbeta", "dS0")]


def load(path: str | None = None):
    """Load (building first if needed) the oracle library; cached per process."""
    global _lib
    with _lock:
        if path is not None:
            lib = ctypes.CDLL(path)
        else:
            if _lib is not None:
                return _lib
            build()
            lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER(_Problem)
        U = ctypes.POINTER(ctypes.c_int64)
        for name in ("gdn_oracle_recurrent", "gdn_oracle_delta_error_form"):
            fn = getattr(lib, name)
            fn.argtypes = [P, U, ctypes.c_int64, ctypes.c_int]
            fn.restype = ctypes.c_int
        lib.gdn_oracle_chunkwise.argtypes = [P, ctypes.POINTER(_ChunkOut), U, ctypes.c_int64, ctypes.c_int]
        lib.gdn_oracle_chunkwise.restype = ctypes.c_int
        lib.gdn_oracle_num_chunks.argtypes = [U, ctypes.c_int64, ctypes.c_int32]
        lib.gdn_oracle_num_chunks.restype = ctypes.c_int64
        D = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_prepare.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           D, D, D, D, ctypes.c_uint32]
        lib.gdn_oracle_prepare.restype = None
        lib.gdn_oracle_output_side.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, D, D, D,
                                               ctypes.c_double, ctypes.c_uint32, D]
        lib.gdn_oracle_output_side.restype = None
        lib.gdn_oracle_short_conv.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, D, D, U,
                                              ctypes.c_int64, D, D, D, ctypes.c_int32]
        lib.gdn_oracle_short_conv.restype = ctypes.c_int
        GP = ctypes.POINTER(_Grads)
        lib.gdn_oracle_backward.argtypes = [P, GP, ctypes.c_int]
        lib.gdn_oracle_backward.restype = ctypes.c_int
        lib.gdn_oracle_backward_chunkwise.argtypes = [P, GP, ctypes.c_int32, ctypes.c_int]
        lib.gdn_oracle_backward_chunkwise.restype = ctypes.c_int
        lib.gdn_oracle_kda_recurrent.argtypes = [P, U, ctypes.c_int64, ctypes.c_int]
        lib.gdn_oracle_kda_recurrent.restype = ctypes.c_int
        lib.gdn_oracle_kda_chunkwise.argtypes = [P, ctypes.c_int32, U, ctypes.c_int64, ctypes.c_int]
        lib.gdn_oracle_kda_chunkwise.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def _dptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _prepare(q, k, v, g, beta, initial_state, cu_seqlens):
    """Accept [B,T,H,d] batched or [T_total,H,d] packed (with cu_seqlens)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    if cu_seqlens is None:
        if q.ndim != 4:
            raise ValueError("batched inputs must be [B, T, H, d]")
        B, T = q.shape[:2]
        cu = np.arange(B + 1, dtype=np.int64) * T
        q, k, v = (x.reshape(B * T, x.shape[2], x.shape[3]) for x in (q, k, v))
        g, beta = (x.reshape(B * T, x.shape[2]) for x in (g, beta))
        batched = (B, T)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        if q.ndim == 4:
            if q.shape[0] != 1:
                raise ValueError("packed inputs need batch 1")
            q, k, v = (x[0] for x in (q, k, v))
            g, beta = (x[0] for x in (g, beta))
            q, k, v, g, beta = (np.ascontiguousarray(x) for x in (q, k, v, g, beta))
            batched = (1, q.shape[0])
        else:
            batched = None
    N = cu.shape[0] - 1
    Ttot, hk, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    if k.shape != q.shape or v.shape[0] != Ttot or g.shape != (Ttot, hv) or beta.shape != (Ttot, hv):
        raise ValueError("shape mismatch")
    if int(cu[-1]) != Ttot:
        raise ValueError("cu_seqlens[-1] must equal the token count")
    s0 = None if initial_state is None else _f64(initial_state).reshape(N, hv, dv, dk)
    return q, k, v, g, beta, s0, cu, batched, (N, Ttot, hk, hv, dk, dv)


def _problem(q, k, v, g, beta, s0, cu, o, sf, dims):
    N, Ttot, hk, hv, dk, dv = dims
    return _Problem(N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), hk, hv, dk, dv,
                    _dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(s0), _dptr(o), _dptr(sf))


def _units_arg(units):
    if units is None:
        return None, ctypes.POINTER(ctypes.c_int64)(), 0
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int64))
    return u, u.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), u.shape[0]


def _finish(o, sf, batched, dims):
    N, Ttot, hk, hv, dk, dv = dims
    if batched is not None:
        B, T = batched
        o = o.reshape(B, T, hv, dv)
    return o, sf


def recurrent(q, k, v, g, beta, initial_state=None, cu_seqlens=None, units=None, threads=None, lib=None):
    """Token recurrence (the oracle proper).  Returns (o, final_state) in fp64.

    ``units`` restricts the work to the listed (sequence * Hv + head) pairs;
    entries of other units are left as NaN so a caller cannot mistake them
    for computed values.
    """
    q, k, v, g, beta, s0, cu, batched, dims = _prepare(q, k, v, g, beta, initial_state, cu_seqlens)
    N, Ttot, hk, hv, dk, dv = dims
    o = np.full((Ttot, hv, dv), np.nan)
    sf = np.full((N, hv, dv, dk), np.nan)
    prob = _problem(q, k, v, g, beta, s0, cu, o, sf, dims)
    keep, uptr, nu = _units_arg(units)
    rc = (lib or load()).gdn_oracle_recurrent(ctypes.byref(prob), uptr, nu, threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle recurrent failed ({rc})")
    return _finish(o, sf, batched, dims)


def delta_error_form(q, k, v, beta, initial_state=None, cu_seqlens=None, threads=None, lib=None):
    """DeltaNet as S <- S - beta (S k - v) k^T, o = S q (no decay gate)."""
    q = _f64(q)
    g = np.zeros(q.shape[:-2] + (np.asarray(v).shape[-2],))
    q, k, v, g, beta, s0, cu, batched, dims = _prepare(q, k, v, g, beta, initial_state, cu_seqlens)
    N, Ttot, hk, hv, dk, dv = dims
    o = np.full((Ttot, hv, dv), np.nan)
    sf = np.full((N, hv, dv, dk), np.nan)
    prob = _problem(q, k, v, g, beta, s0, cu, o, sf, dims)
    rc = (lib or load()).gdn_oracle_delta_error_form(ctypes.byref(prob), None, 0, threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle delta form failed ({rc})")
    return _finish(o, sf, batched, dims)


def chunkwise(q, k, v, g, beta, chunk, initial_state=None, cu_seqlens=None, intermediates=False,
              units=None, threads=None, lib=None):
    """Chunkwise (WY/UT) form in fp64.  Returns (o, final_state[, inter]).

    ``inter`` holds per-chunk arrays indexed [chunk, Hv, ...] (see the C file).
    """
    q, k, v, g, beta, s0, cu, batched, dims = _prepare(q, k, v, g, beta, initial_state, cu_seqlens)
    N, Ttot, hk, hv, dk, dv = dims
    lib = lib or load()
    nch = lib.gdn_oracle_num_chunks(cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, chunk)
    o = np.full((Ttot, hv, dv), np.nan)
    sf = np.full((N, hv, dv, dk), np.nan)
    inter = None
    if intermediates:
        inter = {
            "gcum": np.full((nch, hv, chunk), np.nan),
            "tmat": np.full((nch, hv, chunk, chunk), np.nan),
            "w": np.full((nch, hv, chunk, dk), np.nan),
            "ut": np.full((nch, hv, chunk, dv), np.nan),
            "u": np.full((nch, hv, chunk, dv), np.nan),
            "sc": np.full((nch, hv, dv, dk), np.nan),
        }
    co = _ChunkOut(chunk, *(_dptr(inter[n]) if inter else _dptr(None)
                            for n in ("gcum", "tmat", "w", "ut", "u", "sc")))
    prob = _problem(q, k, v, g, beta, s0, cu, o, sf, dims)
    keep, uptr, nu = _units_arg(units)
    rc = lib.gdn_oracle_chunkwise(ctypes.byref(prob), ctypes.byref(co), uptr, nu, threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle chunkwise failed ({rc})")
    o, sf = _finish(o, sf, batched, dims)
    return (o, sf, inter) if intermediates else (o, sf)


def decode_step(q, k, v, g, beta, state, threads=None, lib=None):
    """One decode token per sequence: q,k [N,Hk,dk], v [N,Hv,dv], g,beta [N,Hv],
    state [N,Hv,dv,dk].  Returns (o [N,Hv,dv], new_state).  This is the token
    recurrence applied to N one-token sequences."""
    N = np.asarray(q).shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return recurrent(q, k, v, g, beta, initial_state=state, cu_seqlens=cu, threads=threads, lib=lib)


def prepare_inputs(q, k, g, beta, qk_l2norm=False, gate_logits=False, lib=None):
    """fp64 copies of q, k, g, beta with the mixer's input side applied
    (``gdn_oracle_prepare``): per-head L2 normalisation of q and k, and the
    decay and write gates from their logits (g = log sigmoid(a),
    beta = sigmoid(b)).  Arrays keep their shapes: q, k [..., Hk, d_k];
    g, beta [..., Hv]."""
    L = lib or load()
    q64, k64 = _f64(q).copy(), _f64(k).copy()
    g64, b64 = _f64(g).copy(), _f64(beta).copy()
    hk, dk = q64.shape[-2], q64.shape[-1]
    hv = g64.shape[-1]
    tokens = q64.size // (hk * dk)
    flags = (2 if qk_l2norm else 0) | (4 if gate_logits else 0)
    L.gdn_oracle_prepare(ctypes.c_int64(tokens), ctypes.c_int32(hk), ctypes.c_int32(hv), ctypes.c_int32(dk),
                         _dptr(q64), _dptr(k64), _dptr(g64), _dptr(b64), ctypes.c_uint32(flags))
    return q64, k64, g64, b64


def short_conv(x, weight, cu_seqlens=None, state=None, silu=True, lib=None):
    """The input side's short causal convolution in fp64
    (``gdn_oracle_short_conv``): one filter of W taps per channel along the
    tokens of each sequence, y[t] = act(sum_j w[j] x[t - (W-1) + j]) with the
    last tap on the current token, then SiLU when ``silu``.

    x is [B, T, *channel dims] (batched) or [T, *channel dims] with
    ``cu_seqlens`` [N + 1]; weight is [*channel dims, W]; state (the W-1
    inputs before each sequence, oldest first) is [N, *channel dims, W-1] or
    None for zeros.  Returns (y shaped like x, the state after each sequence
    [N, *channel dims, W-1])."""
    L = lib or load()
    x64 = _f64(x)
    w64 = _f64(weight)
    width = w64.shape[-1]
    ch_shape = w64.shape[:-1]
    channels = int(np.prod(ch_shape))
    if cu_seqlens is None:
        B, T = x64.shape[0], x64.shape[1]
        assert x64.shape[2:] == ch_shape, (x64.shape, ch_shape)
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        assert x64.shape[1:] == ch_shape, (x64.shape, ch_shape)
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = cu.shape[0] - 1
    tokens = x64.size // channels
    s64 = None
    if state is not None:
        s64 = _f64(state)
        assert s64.shape == (n, *ch_shape, width - 1), (s64.shape, (n, *ch_shape, width - 1))
    y = np.empty_like(x64)
    s_out = np.empty((n, *ch_shape, width - 1))
    rc = L.gdn_oracle_short_conv(ctypes.c_int64(tokens), ctypes.c_int32(channels), ctypes.c_int32(width),
                                 _dptr(x64), _dptr(w64), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 ctypes.c_int64(n), _dptr(s64), _dptr(y), _dptr(s_out),
                                 ctypes.c_int32(1 if silu else 0))
    if rc != 0:
        raise ValueError("oracle short_conv rejected its arguments")
    return y, s_out


# output-side flags of gdn_oracle_output_side (the oracle's own numbering)
OUT_GATE_SILU, OUT_GATE_SIGMOID, OUT_ZERO_CENTRED, OUT_WEIGHT_PER_HEAD = 1, 2, 4, 8


def output_side(o, z=None, weight=None, eps=1e-6, gate="silu", zero_centred=False, lib=None):
    """The mixer's output side on o [..., Hv, d_v] in fp64
    (``gdn_oracle_output_side``): each (token, value head) row divided by
    its root mean square (+ eps inside the root), times the scale (w, or
    1 + w when zero_centred; weight [d_v] shared by the heads or [Hv, d_v]
    per head), times act(z) with act = SiLU or sigmoid (``gate``) when z is
    given.  Returns a new array of o's shape."""
    L = lib or load()
    o64 = _f64(o).copy()
    hv, dv = o64.shape[-2], o64.shape[-1]
    tokens = o64.size // (hv * dv)
    flags = 0
    z64 = None
    if z is not None:
        z64 = _f64(z).copy()
        assert z64.shape == o64.shape
        flags |= {"silu": OUT_GATE_SILU, "sigmoid": OUT_GATE_SIGMOID}[gate]
    w64 = None
    if weight is not None:
        w64 = _f64(weight).copy()
        if w64.ndim == 2:
            assert w64.shape == (hv, dv)
            flags |= OUT_WEIGHT_PER_HEAD
        else:
            assert w64.shape == (dv,)
    if zero_centred:
        flags |= OUT_ZERO_CENTRED
    y = np.empty_like(o64)
    L.gdn_oracle_output_side(ctypes.c_int64(tokens), ctypes.c_int32(hv), ctypes.c_int32(dv), _dptr(o64),
                             _dptr(z64), _dptr(w64), ctypes.c_double(eps), ctypes.c_uint32(flags), _dptr(y))
    return y


def _kda_run(name, q, k, v, g, beta, initial_state, cu_seqlens, units, threads, lib, extra=()):
    """KDA: g holds one log-decay per key channel, [..., Hv, d_k]."""
    g64 = _f64(g)
    q, k, v, g0, beta, s0, cu, batched, dims = _prepare(q, k, v, g64[..., 0], beta, initial_state, cu_seqlens)
    N, Ttot, hk, hv, dk, dv = dims
    gk = np.ascontiguousarray(g64.reshape(Ttot, hv, dk))
    o = np.full((Ttot, hv, dv), np.nan)
    sf = np.full((N, hv, dv, dk), np.nan)
    prob = _problem(q, k, v, gk, beta, s0, cu, o, sf, dims)
    keep, uptr, nu = _units_arg(units)
    fn = getattr(lib or load(), name)
    rc = fn(ctypes.byref(prob), *extra, uptr, nu, threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle {name} failed ({rc})")
    return _finish(o, sf, batched, dims)


def kda_recurrent(q, k, v, g, beta, initial_state=None, cu_seqlens=None, units=None, threads=None, lib=None):
    """Kimi Delta Attention, token recurrence (``gdn_oracle_kda_recurrent``):
    g [..., Hv, d_k] is the per-key-channel log-decay.  Returns (o, final_state)."""
    return _kda_run("gdn_oracle_kda_recurrent", q, k, v, g, beta, initial_state, cu_seqlens, units, threads, lib)


def kda_chunkwise(q, k, v, g, beta, chunk, initial_state=None, cu_seqlens=None, units=None, threads=None, lib=None):
    """Kimi Delta Attention in chunks of ``chunk`` tokens (``gdn_oracle_kda_chunkwise``),
    an independent formulation derived from the recurrence."""
    return _kda_run("gdn_oracle_kda_chunkwise", q, k, v, g, beta, initial_state, cu_seqlens, units, threads, lib,
                    extra=(ctypes.c_int32(chunk),))


def kda_decode_step(q, k, v, g, beta, state, threads=None, lib=None):
    """One KDA token per sequence: q,k [N,Hk,dk], v [N,Hv,dv], g [N,Hv,dk],
    beta [N,Hv], state [N,Hv,dv,dk].  Returns (o, new_state)."""
    N = np.asarray(q).shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return kda_recurrent(q, k, v, g, beta, initial_state=state, cu_seqlens=cu, threads=threads, lib=lib)


def prepare_kda_inputs(q, k, g, beta, qk_l2norm=False, gate_logits=False, lib=None):
    """The input side for KDA: as ``prepare_inputs``, with g [..., Hv, d_k]
    holding one logit per key channel (each becomes log sigmoid of itself;
    the transform is elementwise, so the channels pass as extra heads)."""
    q64, k64, _, b64 = prepare_inputs(q, k, np.zeros_like(_f64(beta)), beta, qk_l2norm=qk_l2norm,
                                      gate_logits=gate_logits, lib=lib)
    g64 = _f64(g).copy()
    if gate_logits:
        flat = g64.reshape(-1, g64.shape[-2] * g64.shape[-1])
        _, _, gp, _ = prepare_inputs(np.zeros((flat.shape[0], 1, 1)), np.zeros((flat.shape[0], 1, 1)), flat,
                                     np.zeros_like(flat), gate_logits=True, lib=lib)
        g64 = gp.reshape(g64.shape)
    return q64, k64, g64, b64


def conv_input_side(q, k, v, conv_q, conv_k, conv_v, cu_seqlens=None, states=None, lib=None):
    """The input side up to the recurrence's q, k and v, as "Architecture
    Thread I" ("Modern Architecture Improvements") orders it: q and k pass
    through the short causal convolution, SiLU and per-head L2
    normalisation; v through the short convolution and SiLU.  A composition
    of ``short_conv`` and ``prepare_inputs`` (both pinned), no arithmetic of
    its own.  conv_q, conv_k are [Hk, d_k, W] and conv_v [Hv, d_v, W];
    ``states`` is None or a dict of conv states {"q", "k", "v"} each
    [N, H, d, W-1].  Returns (q, k, v, the conv states after each sequence)."""
    st = states or {}
    cq, sq = short_conv(q, conv_q, cu_seqlens=cu_seqlens, state=st.get("q"), silu=True, lib=lib)
    ck, sk = short_conv(k, conv_k, cu_seqlens=cu_seqlens, state=st.get("k"), silu=True, lib=lib)
    cv, sv = short_conv(v, conv_v, cu_seqlens=cu_seqlens, state=st.get("v"), silu=True, lib=lib)
    lead = cq.shape[:-2]
    zeros = np.zeros(lead + (1,))
    qn, kn, _, _ = prepare_inputs(cq, ck, zeros, zeros, qk_l2norm=True, lib=lib)
    return qn, kn, cv, {"q": sq, "k": sk, "v": sv}


def decode_multi(q, k, v, g, beta, state, threads=None, lib=None):
    """K decode tokens per sequence with the state after every token:
    q, k [N, K, Hk, dk], v [N, K, Hv, dv], g, beta [N, K, Hv], state
    [N, Hv, dv, dk].  Returns (o [N, K, Hv, dv], snapshots [N, K, Hv, dv, dk]).
    A composition of ``decode_step`` (the pinned token recurrence), one token
    at a time; no arithmetic of its own."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S = _f64(state).copy()
    N, K = q.shape[:2]
    o = np.empty(v.shape)
    snaps = np.empty((N, K) + S.shape[1:])
    for j in range(K):
        o[:, j], S = decode_step(q[:, j], k[:, j], v[:, j], g[:, j], beta[:, j], S, threads=threads, lib=lib)
        snaps[:, j] = S
    return o, snaps


def backward(q, k, v, g, beta, dO, dS_final=None, initial_state=None, cu_seqlens=None, chunk=None, threads=None,
             lib=None):
    """Gradients of L = sum dO . o + sum dS_final . S_final with respect to
    q, k, v, g, beta and the initial state (``gdn_oracle_backward``: reverse
    mode of the token recurrence; with ``chunk``: ``gdn_oracle_backward_chunkwise``,
    the chunked form differentiated).  Returns a dict of fp64 arrays shaped
    like the inputs: dq, dk (summed over the value heads of each q/k group),
    dv, dg, dbeta, dS0."""
    q, k, v, g, beta, s0, cu, batched, dims = _prepare(q, k, v, g, beta, initial_state, cu_seqlens)
    N, Ttot, hk, hv, dk, dv = dims
    dO64 = np.ascontiguousarray(_f64(dO).reshape(Ttot, hv, dv))
    dSf = None if dS_final is None else np.ascontiguousarray(_f64(dS_final).reshape(N, hv, dv, dk))
    out = {"dq": np.zeros((Ttot, hv, dk)), "dk": np.zeros((Ttot, hv, dk)), "dv": np.zeros((Ttot, hv, dv)),
           "dg": np.zeros((Ttot, hv)), "dbeta": np.zeros((Ttot, hv)), "dS0": np.zeros((N, hv, dv, dk))}
    gr = _Grads(_dptr(dO64), _dptr(dSf), _dptr(out["dq"]), _dptr(out["dk"]), _dptr(out["dv"]), _dptr(out["dg"]),
                _dptr(out["dbeta"]), _dptr(out["dS0"]))
    prob = _problem(q, k, v, g, beta, s0, cu, None, None, dims)
    L = lib or load()
    if chunk is None:
        rc = L.gdn_oracle_backward(ctypes.byref(prob), ctypes.byref(gr), threads or default_threads())
    else:
        rc = L.gdn_oracle_backward_chunkwise(ctypes.byref(prob), ctypes.byref(gr), ctypes.c_int32(chunk),
                                             threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle backward failed ({rc})")
    G = hv // hk
    for n in ("dq", "dk"):
        out[n] = out[n].reshape(Ttot, hk, G, dk).sum(axis=2)
    if batched is not None:
        B, T = batched
        out["dq"] = out["dq"].reshape(B, T, hk, dk)
        out["dk"] = out["dk"].reshape(B, T, hk, dk)
        out["dv"] = out["dv"].reshape(B, T, hv, dv)
        out["dg"] = out["dg"].reshape(B, T, hv)
        out["dbeta"] = out["dbeta"].reshape(B, T, hv)
    return out

