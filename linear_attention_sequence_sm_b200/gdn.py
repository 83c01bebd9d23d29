"""Python binding of libgdn.so (the gated delta rule on B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/gdn.h``.  PyTorch provides
device memory and streams.  There is no CPU fallback: if the library is
missing, importing this module raises.

Layouts (row-major, token-major):
  q, k  [B, T, Hk, d_k] (or [T, Hk, d_k] packed with cu_seqlens)
  v, o  [B, T, Hv, d_v]
  g, beta [B, T, Hv] fp32;  states [N, Hv, d_v, d_k] fp32
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARGUMENT = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_MISALIGNED = 3
GDN_ERR_WORKSPACE_TOO_SMALL = 4
GDN_ERR_CUDA = 5
GDN_ERR_DEVICE_CHECK = 6
GDN_DTYPE_F32 = 0
GDN_DTYPE_BF16 = 1
GDN_FLAG_FORCE_SIMT = 1
GDN_FLAG_QK_L2NORM = 2
GDN_FLAG_GATE_LOGITS = 4
GDN_FLAG_ONE_KERNEL = 8
GDN_FLAG_SPLIT = 16
GDN_OUT_GATE_SILU = 1
GDN_OUT_GATE_SIGMOID = 2
GDN_OUT_ZERO_CENTRED = 4
GDN_OUT_WEIGHT_PER_HEAD = 8
GDN_CONV_SILU = 1

EXPORTED = ("gdn_chunk_forward_workspace_size", "gdn_chunk_forward", "gdn_read_device_status",
            "gdn_decode_step", "gdn_status_string", "gdn_last_error_message", "gdn_launch_count",
            "gdn_chunk_forward_noalloc", "gdn_decode_step_ex", "gdn_chunk_forward_out", "gdn_decode_step_out",
            "gdn_kda_forward", "gdn_kda_decode_step", "gdn_decode_multi", "gdn_decode_commit",
            "gdn_chunk_backward_workspace_size", "gdn_chunk_backward", "gdn_short_conv",
            "gdn_chunk_forward_path", "gdn_noalloc_read_device_status", "gdn_kda_forward_workspace_size")
GDN_PATH_SIMT = 0
GDN_PATH_TC_ONE_KERNEL = 1
GDN_PATH_TC_SPLIT = 2
PATH_NAMES = {GDN_PATH_SIMT: "simt", GDN_PATH_TC_ONE_KERNEL: "tc_one_kernel", GDN_PATH_TC_SPLIT: "tc_split"}


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} [status {status}]")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("num_qk_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_dim_k", ctypes.c_int32), ("head_dim_v", ctypes.c_int32),
                ("chunk_size", ctypes.c_int32), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class OutputSideC(ctypes.Structure):
    _fields_ = [("weight", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"libgdn.so not found at {path}; build it with "
                          "`python -m linear_attention_sequence_sm_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int
    lib.gdn_chunk_forward_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)]
    lib.gdn_chunk_forward_workspace_size.restype = st
    lib.gdn_chunk_forward_path.argtypes = [ctypes.POINTER(Shape), ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)]
    lib.gdn_chunk_forward_path.restype = st
    lib.gdn_kda_forward_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)]
    lib.gdn_kda_forward_workspace_size.restype = st
    lib.gdn_noalloc_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    lib.gdn_noalloc_read_device_status.restype = st
    lib.gdn_chunk_forward.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      ctypes.c_size_t, vp]
    lib.gdn_chunk_forward.restype = st
    lib.gdn_chunk_forward_noalloc.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_chunk_forward_noalloc.restype = st
    lib.gdn_read_device_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    lib.gdn_read_device_status.restype = st
    lib.gdn_decode_step.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_decode_step.restype = st
    lib.gdn_decode_step_ex.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, ctypes.c_uint32, vp]
    lib.gdn_decode_step_ex.restype = st
    osp = ctypes.POINTER(OutputSideC)
    lib.gdn_chunk_forward_out.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, osp, vp, vp, vp,
                                          ctypes.c_size_t, vp]
    lib.gdn_chunk_forward_out.restype = st
    lib.gdn_decode_step_out.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, osp, vp,
                                        ctypes.c_uint32, vp]
    lib.gdn_decode_step_out.restype = st
    lib.gdn_kda_forward.argtypes = lib.gdn_chunk_forward_out.argtypes
    lib.gdn_kda_forward.restype = st
    lib.gdn_kda_decode_step.argtypes = lib.gdn_decode_step_out.argtypes
    lib.gdn_kda_decode_step.restype = st
    lib.gdn_decode_multi.argtypes = [i32] * 7 + [vp] * 8 + [ctypes.c_uint32, vp]
    lib.gdn_decode_multi.restype = st
    lib.gdn_decode_commit.argtypes = [i32] * 5 + [vp] * 4 + [vp]
    lib.gdn_decode_commit.restype = st
    lib.gdn_chunk_backward_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)]
    lib.gdn_chunk_backward_workspace_size.restype = st
    lib.gdn_chunk_backward.argtypes = [ctypes.POINTER(Shape)] + [vp] * 15 + [vp, ctypes.c_size_t, vp]
    lib.gdn_chunk_backward.restype = st
    lib.gdn_short_conv.argtypes = [i32, i32, vp, ctypes.c_int64, i32, i32, i32, vp, vp, vp, vp, vp,
                                   ctypes.c_uint32, vp]
    lib.gdn_short_conv.restype = st
    lib.gdn_status_string.argtypes = [st]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_last_error_message.argtypes = []
    lib.gdn_last_error_message.restype = ctypes.c_char_p
    lib.gdn_launch_count.argtypes = []
    lib.gdn_launch_count.restype = ctypes.c_uint64
    return lib


LIB = _load()


def _check(status: int):
    if status != GDN_OK:
        name = LIB.gdn_status_string(status).decode()
        raise GdnError(status, f"{name}: {LIB.gdn_last_error_message().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_DTYPE_BF16
    if t.dtype == torch.float32:
        return GDN_DTYPE_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _stream_handle(stream, dev):
    """The stream a call enqueues on: ``stream``, or the current stream of the
    tensors' device ``dev``.  A stream of another device is rejected: the
    library would launch on it with pointers into ``dev``'s memory."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _expect(t, name, shape):
    """``t`` (if given) must have exactly ``shape``: the library takes bare
    pointers and derives every extent from q and v, so a tensor of another
    shape would be read or written out of bounds on the device."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _prefill_shapes(q, k, v, g, beta, initial_state, cu_seqlens, kda=False):
    """Shape checks of the prefill and backward inputs (before any device
    check, so they hold for tensors anywhere).  Returns (N, Hv, d_v, d_k)."""
    if cu_seqlens is not None:
        if q.dim() not in (3, 4) or (q.dim() == 4 and q.shape[0] != 1):
            raise ValueError(f"with cu_seqlens q must be [T, Hk, d_k] or [1, T, Hk, d_k], got {tuple(q.shape)}")
        if cu_seqlens.dim() != 1 or cu_seqlens.shape[0] < 1:
            raise ValueError(f"cu_seqlens must be [N + 1], got {tuple(cu_seqlens.shape)}")
        n_seqs = cu_seqlens.shape[0] - 1
    else:
        if q.dim() != 4:
            raise ValueError(f"batched q must be [B, T, Hk, d_k], got {tuple(q.shape)}")
        n_seqs = q.shape[0]
    _expect(k, "k", q.shape)
    if v.dim() != q.dim() or tuple(v.shape[:-2]) != tuple(q.shape[:-2]):
        raise ValueError(f"v must be [{', '.join(map(str, q.shape[:-2]))}, Hv, d_v], got {tuple(v.shape)}")
    hv, dv, dk = v.shape[-2], v.shape[-1], q.shape[-1]
    _expect(g, "g", tuple(v.shape[:-1]) + ((dk,) if kda else ()))
    _expect(beta, "beta", v.shape[:-1])
    _expect(initial_state, "initial_state", (n_seqs, hv, dv, dk))
    return n_seqs, hv, dv, dk


def _decode_shapes(q, k, v, g, beta, state, kda=False):
    """Shape checks of one decode step: q, k [N, Hk, d_k], v [N, Hv, d_v],
    g [N, Hv] ([N, Hv, d_k] for KDA), beta [N, Hv], state [N, Hv, d_v, d_k]."""
    if q.dim() != 3:
        raise ValueError(f"decode q must be [N, Hk, d_k], got {tuple(q.shape)}")
    _expect(k, "k", q.shape)
    if v.dim() != 3 or v.shape[0] != q.shape[0]:
        raise ValueError(f"decode v must be [{q.shape[0]}, Hv, d_v], got {tuple(v.shape)}")
    n, hv, dv, dk = q.shape[0], v.shape[1], v.shape[2], q.shape[2]
    _expect(g, "g", (n, hv, dk) if kda else (n, hv))
    _expect(beta, "beta", (n, hv))
    _expect(state, "state", (n, hv, dv, dk))


def input_flags(qk_l2norm=False, gate_logits=False) -> int:
    """GDN_FLAG_QK_L2NORM / GDN_FLAG_GATE_LOGITS bits: raw q and k normalised
    per head inside the kernels; g and beta given as logits."""
    return (GDN_FLAG_QK_L2NORM if qk_l2norm else 0) | (GDN_FLAG_GATE_LOGITS if gate_logits else 0)


class OutputNorm:
    """The mixer's output side, applied in the kernels to every (token, value
    head) output row o: y = o / sqrt(mean(o^2) + eps) * s * act(gate).

    weight        fp32 [d_v] (shared by the value heads) or [Hv, d_v], or None
                  for a unit scale; with ``zero_centred`` the scale is
                  1 + weight.
    gate          the gate pre-activation z, shaped and typed like o, or None.
    activation    "silu" (z * sigmoid(z)) or "sigmoid" (used with a gate).
    """

    def __init__(self, weight=None, gate=None, eps=1e-6, activation="silu", zero_centred=False):
        if activation not in ("silu", "sigmoid"):
            raise ValueError(f"activation must be 'silu' or 'sigmoid', got {activation!r}")
        self.weight, self.gate, self.eps = weight, gate, float(eps)
        self.activation, self.zero_centred = activation, bool(zero_centred)

    def c_struct(self, o: torch.Tensor) -> OutputSideC:
        hv, dv = o.shape[-2], o.shape[-1]
        flags = GDN_OUT_ZERO_CENTRED if self.zero_centred else 0
        if self.weight is not None:
            _need(self.weight, "output weight", torch.float32, o.device)
            if tuple(self.weight.shape) == (hv, dv):
                flags |= GDN_OUT_WEIGHT_PER_HEAD
            elif tuple(self.weight.shape) != (dv,):
                raise ValueError(f"output weight must be [{dv}] or [{hv}, {dv}], got {tuple(self.weight.shape)}")
        if self.gate is not None:
            _need(self.gate, "output gate", o.dtype, o.device)
            if self.gate.shape != o.shape:
                raise ValueError(f"output gate must have o's shape {tuple(o.shape)}, got {tuple(self.gate.shape)}")
            flags |= GDN_OUT_GATE_SILU if self.activation == "silu" else GDN_OUT_GATE_SIGMOID
        return OutputSideC(None if self.weight is None else self.weight.data_ptr(),
                           None if self.gate is None else self.gate.data_ptr(), self.eps, flags)


def make_shape(q, v, cu_seqlens=None, chunk_size=64, force_simt=False, flags=0, one_kernel=False,
               split=False) -> Shape:
    if cu_seqlens is not None:
        T = q.shape[-3]
        B, N = 1, cu_seqlens.shape[0] - 1
    else:
        if q.dim() != 4:
            raise ValueError("batched q must be [B, T, Hk, d_k]")
        B, T = q.shape[0], q.shape[1]
        N = B
    return Shape(B, T, N, q.shape[-2], v.shape[-2], q.shape[-1], v.shape[-1], chunk_size, _dtype_code(q),
                 (GDN_FLAG_FORCE_SIMT if force_simt else 0) | (GDN_FLAG_ONE_KERNEL if one_kernel else 0) |
                 (GDN_FLAG_SPLIT if split else 0) | flags)


def forward_path(shape: Shape, workspace_bytes: int | None = None) -> str:
    """The kernel path gdn_chunk_forward takes for ``shape`` on the current
    device ("simt", "tc_one_kernel" or "tc_split"), with a workspace of
    ``workspace_bytes`` (default: the queried size)."""
    if workspace_bytes is None:
        workspace_bytes = workspace_size(shape)
    p = ctypes.c_int32(-1)
    _check(LIB.gdn_chunk_forward_path(ctypes.byref(shape), ctypes.c_size_t(workspace_bytes), ctypes.byref(p)))
    return PATH_NAMES[p.value]


def kda_workspace_size(shape: Shape) -> int:
    """Bytes of workspace gdn_kda_forward needs for ``shape``."""
    n = ctypes.c_size_t(0)
    _check(LIB.gdn_kda_forward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(LIB.gdn_chunk_forward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def chunk_forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk_size=64,
                  output_final_state=True, out=None, final_state=None, workspace=None, force_simt=False,
                  stream=None, qk_l2norm=False, gate_logits=False, output_norm: OutputNorm | None = None,
                  one_kernel=False, split=False):
    """Chunkwise prefill.  Returns (o, final_state or None).  Asynchronous on
    ``stream`` (default: the current stream).  ``qk_l2norm``: q and k are raw
    and normalised per head in the kernel; ``gate_logits``: g and beta are
    the decay and write logits (alpha = sigmoid(g), beta = sigmoid(beta));
    ``output_norm``: the output side applied before o is stored;
    ``one_kernel``: never the two-kernel tensor-core form (GDN_FLAG_ONE_KERNEL,
    schedule-sized workspace); ``split``: the two-kernel form wherever it
    applies (GDN_FLAG_SPLIT)."""
    n_seqs, hv, dv, dk = _prefill_shapes(q, k, v, g, beta, initial_state, cu_seqlens)
    _expect(out, "out", v.shape)
    _expect(final_state, "final_state", (n_seqs, hv, dv, dk))
    dev = q.device
    dt = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(initial_state, "initial_state", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    shape = make_shape(q, v, cu_seqlens, chunk_size, force_simt, input_flags(qk_l2norm, gate_logits), one_kernel,
                       split)
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    _need(out, "out", dt, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((shape.num_seqs, shape.num_v_heads, shape.head_dim_v, shape.head_dim_k),
                                  dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev)
    nbytes = workspace_size(shape)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if output_norm is not None:
        osc = output_norm.c_struct(out)
        with torch.cuda.device(dev):  # the library launches on the current device
            _check(LIB.gdn_chunk_forward_out(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                             _ptr(initial_state), _ptr(cu_seqlens), ctypes.byref(osc), _ptr(out),
                                             _ptr(final_state), _ptr(workspace), workspace.numel(),
                                             _stream_handle(stream, dev)))
        return out, final_state
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_chunk_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                     _ptr(initial_state), _ptr(cu_seqlens), _ptr(out), _ptr(final_state),
                                     _ptr(workspace), workspace.numel(), _stream_handle(stream, dev)))
    return out, final_state


def chunk_forward_noalloc(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk_size=64,
                          output_final_state=True, out=None, final_state=None, force_simt=False, stream=None,
                          qk_l2norm=False, gate_logits=False):
    """chunk_forward for callers that cannot allocate device scratch: the
    library's built-in scratch array stands in for the workspace (at most
    16,384 sequences; calls that overlap on the GPU race on that array).
    Output tensors are still the caller's (allocated here only when not
    given)."""
    n_seqs, hv, dv, dk = _prefill_shapes(q, k, v, g, beta, initial_state, cu_seqlens)
    _expect(out, "out", v.shape)
    _expect(final_state, "final_state", (n_seqs, hv, dv, dk))
    dev = q.device
    dt = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(initial_state, "initial_state", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    shape = make_shape(q, v, cu_seqlens, chunk_size, force_simt, input_flags(qk_l2norm, gate_logits))
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    _need(out, "out", dt, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((shape.num_seqs, shape.num_v_heads, shape.head_dim_v, shape.head_dim_k),
                                  dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev)
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_chunk_forward_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                             _ptr(initial_state), _ptr(cu_seqlens), _ptr(out), _ptr(final_state),
                                             _stream_handle(stream, dev)))
    return out, final_state


def read_device_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the device status word of the last
    gdn_chunk_forward that used ``workspace``."""
    st = ctypes.c_int32(-1)
    dev = workspace.device
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_read_device_status(_ptr(workspace), ctypes.byref(st), _stream_handle(stream, dev)))
    return st.value


def noalloc_read_device_status(device=None, stream=None) -> int:
    """Synchronise the stream and return the device status word of the last
    gdn_chunk_forward_noalloc on ``device`` (default: the current device)."""
    st = ctypes.c_int32(-1)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(LIB.gdn_noalloc_read_device_status(ctypes.byref(st), _stream_handle(stream, dev)))
    return st.value


def decode_step(q, k, v, g, beta, state, out=None, stream=None, qk_l2norm=False, gate_logits=False,
                output_norm: OutputNorm | None = None):
    """One token per sequence; ``state`` [N, Hv, d_v, d_k] fp32 is updated in
    place.  Returns o [N, Hv, d_v].  ``qk_l2norm``, ``gate_logits`` and
    ``output_norm`` (gate [N, Hv, d_v]) as for chunk_forward."""
    _decode_shapes(q, k, v, g, beta, state)
    _expect(out, "out", v.shape)
    dev, dt = q.device, q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    _need(out, "out", dt, dev)
    N, hk, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    if output_norm is not None:
        osc = output_norm.c_struct(out)
        with torch.cuda.device(dev):  # the library launches on the current device
            _check(LIB.gdn_decode_step_out(N, hk, hv, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                           _ptr(beta), _ptr(state), ctypes.byref(osc), _ptr(out),
                                           input_flags(qk_l2norm, gate_logits), _stream_handle(stream, dev)))
        return out
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_decode_step_ex(N, hk, hv, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                      _ptr(beta), _ptr(state), _ptr(out), input_flags(qk_l2norm, gate_logits),
                                      _stream_handle(stream, dev)))
    return out


def kda_forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, output_final_state=True, out=None,
                final_state=None, workspace=None, stream=None, qk_l2norm=False, gate_logits=False,
                output_norm: OutputNorm | None = None, chunk_size=64, force_simt=False):
    """Kimi Delta Attention prefill (one decay per key channel): g is
    [..., Hv, d_k] fp32.  Returns (o, final_state or None).  Other arguments
    as for chunk_forward.  bf16 with d = 128 and chunk_size 64 runs the
    tensor-core chunkwise form; other shapes, or ``force_simt``, the
    token-order CUDA-core kernel."""
    n_seqs, hv, dv, dk = _prefill_shapes(q, k, v, g, beta, initial_state, cu_seqlens, kda=True)
    _expect(out, "out", v.shape)
    _expect(final_state, "final_state", (n_seqs, hv, dv, dk))
    dev = q.device
    dt = q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(initial_state, "initial_state", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    shape = make_shape(q, v, cu_seqlens, chunk_size, force_simt, input_flags(qk_l2norm, gate_logits))
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    _need(out, "out", dt, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((shape.num_seqs, shape.num_v_heads, shape.head_dim_v, shape.head_dim_k),
                                  dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev)
    nbytes = kda_workspace_size(shape)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    osc = output_norm.c_struct(out) if output_norm is not None else None
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_kda_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(initial_state), _ptr(cu_seqlens), None if osc is None else ctypes.byref(osc),
                                   _ptr(out), _ptr(final_state), _ptr(workspace), workspace.numel(),
                                   _stream_handle(stream, dev)))
    return out, final_state


def kda_decode_step(q, k, v, g, beta, state, out=None, stream=None, qk_l2norm=False, gate_logits=False,
                    output_norm: OutputNorm | None = None):
    """One Kimi Delta Attention token per sequence: g [N, Hv, d_k] fp32;
    ``state`` [N, Hv, d_v, d_k] fp32 updated in place.  Returns o [N, Hv, d_v]."""
    _decode_shapes(q, k, v, g, beta, state, kda=True)
    _expect(out, "out", v.shape)
    dev, dt = q.device, q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    N, hk, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    _need(out, "out", dt, dev)
    osc = output_norm.c_struct(out) if output_norm is not None else None
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_kda_decode_step(N, hk, hv, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                       _ptr(beta), _ptr(state), None if osc is None else ctypes.byref(osc), _ptr(out),
                                       input_flags(qk_l2norm, gate_logits), _stream_handle(stream, dev)))
    return out


def decode_multi(q, k, v, g, beta, state, out=None, snapshots=None, stream=None, qk_l2norm=False,
                 gate_logits=False):
    """K decode tokens per sequence in one pass (draft verification): q, k
    [N, K, Hk, 128], v [N, K, Hv, d_v], g, beta [N, K, Hv]; ``state``
    [N, Hv, d_v, 128] fp32 is only read.  Returns (o [N, K, Hv, d_v],
    snapshots [N, K, Hv, d_v, 128] fp32: the state after each token)."""
    if q.dim() != 4:
        raise ValueError(f"multi-token decode q must be [N, K, Hk, d_k], got {tuple(q.shape)}")
    _expect(k, "k", q.shape)
    if v.dim() != 4 or tuple(v.shape[:2]) != tuple(q.shape[:2]):
        raise ValueError(f"v must be [{q.shape[0]}, {q.shape[1]}, Hv, d_v], got {tuple(v.shape)}")
    n_, k_, hv_, dv_, dk_ = q.shape[0], q.shape[1], v.shape[2], v.shape[3], q.shape[3]
    _expect(g, "g", (n_, k_, hv_))
    _expect(beta, "beta", (n_, k_, hv_))
    _expect(state, "state", (n_, hv_, dv_, dk_))
    _expect(out, "out", v.shape)
    _expect(snapshots, "snapshots", (n_, k_, hv_, dv_, dk_))
    dev, dt = q.device, q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    N, K, hk, dk = q.shape
    hv, dv = v.shape[2], v.shape[3]
    if out is None:
        out = torch.empty(v.shape, dtype=dt, device=dev)
    if snapshots is None:
        snapshots = torch.empty((N, K, hv, dv, dk), dtype=torch.float32, device=dev)
    _need(out, "out", dt, dev)
    _need(snapshots, "snapshots", torch.float32, dev)
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_decode_multi(N, K, hk, hv, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                    _ptr(beta), _ptr(state), _ptr(snapshots), _ptr(out),
                                    input_flags(qk_l2norm, gate_logits), _stream_handle(stream, dev)))
    return out, snapshots


def decode_commit(snapshots, accepted, state, bad_count=None, stream=None):
    """state[n] <- snapshots[n, accepted[n] - 1] for accepted[n] in 1..K
    (0 keeps state[n]); ``accepted`` int32 [N] on the device."""
    if snapshots.dim() != 5:
        raise ValueError(f"snapshots must be [N, K, Hv, d_v, d_k], got {tuple(snapshots.shape)}")
    n_, _, hv_, dv_, dk_ = snapshots.shape
    _expect(accepted, "accepted", (n_,))
    _expect(state, "state", (n_, hv_, dv_, dk_))
    if bad_count is not None and bad_count.numel() < 1:
        raise ValueError("bad_count must hold at least one int32")
    dev = state.device
    _need(snapshots, "snapshots", torch.float32, dev)
    _need(accepted, "accepted", torch.int32, dev)
    _need(state, "state", torch.float32, dev)
    _need(bad_count, "bad_count", torch.int32, dev)
    N, K, hv, dv, dk = snapshots.shape
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_decode_commit(N, K, hv, dk, dv, _ptr(snapshots), _ptr(accepted), _ptr(state), _ptr(bad_count),
                                     _stream_handle(stream, dev)))
    return state


def chunk_backward(q, k, v, g, beta, d_o, d_final_state=None, initial_state=None, cu_seqlens=None,
                   want_d_initial_state=True, workspace=None, stream=None, force_simt=False):
    """Gradients of sum d_o . o + sum d_final_state . S_final (training).
    Returns a dict of fp32 tensors: dq, dk (shaped like q), dv (like v),
    dg, dbeta (like g), d_initial_state ([N, Hv, d_v, d_k], or None).
    bf16 inputs with d_k = d_v = 128 take the tensor-core kernels on sm_100
    unless ``force_simt`` (GDN_FLAG_FORCE_SIMT) picks the single-kernel form."""
    n_seqs, hv, dv, dk = _prefill_shapes(q, k, v, g, beta, initial_state, cu_seqlens)
    _expect(d_o, "d_o", v.shape)
    _expect(d_final_state, "d_final_state", (n_seqs, hv, dv, dk))
    dev, dt = q.device, q.dtype
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o")):
        _need(t, n, dt, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(initial_state, "initial_state", torch.float32, dev)
    _need(d_final_state, "d_final_state", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    shape = make_shape(q, v, cu_seqlens, 32, force_simt=force_simt)
    n = ctypes.c_size_t(0)
    _check(LIB.gdn_chunk_backward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    if workspace is None or workspace.numel() < n.value:
        workspace = torch.empty(n.value, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32), "dv": torch.empty(v.shape, **f32),
           "dg": torch.empty(g.shape, **f32), "dbeta": torch.empty(beta.shape, **f32),
           "d_initial_state": torch.empty((shape.num_seqs, shape.num_v_heads, shape.head_dim_v, shape.head_dim_k),
                                          **f32) if want_d_initial_state else None}
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_chunk_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                      _ptr(initial_state), _ptr(cu_seqlens), _ptr(d_o), _ptr(d_final_state),
                                      _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                      _ptr(out["dbeta"]), _ptr(out["d_initial_state"]), _ptr(workspace),
                                      workspace.numel(), _stream_handle(stream, dev)))
    return out


def short_conv(x, weight, cu_seqlens=None, state=None, silu=True, out=None, state_out=None,
               want_state=True, stream=None):
    """The input side's short causal convolution (depthwise, W taps per
    channel, the last on the current token), then SiLU when ``silu``.
    x is [B, T, *channel dims] (batched) or [T, *channel dims] /
    [1, T, *channel dims] with ``cu_seqlens``; weight [*channel dims, W]
    fp32; state (each sequence's W-1 preceding inputs, oldest first)
    [N, *channel dims, W-1] fp32 or None for zeros.  Returns (y shaped like
    x, the state after each sequence or None)."""
    if weight.dim() < 2:
        raise ValueError(f"weight must be [*channel dims, W], got {tuple(weight.shape)}")
    ch = tuple(weight.shape[:-1])
    width = weight.shape[-1]
    nch = len(ch)
    if cu_seqlens is not None:
        if x.dim() not in (nch + 1, nch + 2) or (x.dim() == nch + 2 and x.shape[0] != 1):
            raise ValueError(f"with cu_seqlens x must be [T, *{ch}] or [1, T, *{ch}], got {tuple(x.shape)}")
        if cu_seqlens.dim() != 1 or cu_seqlens.shape[0] < 1:
            raise ValueError(f"cu_seqlens must be [N + 1], got {tuple(cu_seqlens.shape)}")
        n_seqs, seq_len = cu_seqlens.shape[0] - 1, 0
    else:
        if x.dim() != nch + 2:
            raise ValueError(f"batched x must be [B, T, *{ch}], got {tuple(x.shape)}")
        n_seqs, seq_len = x.shape[0], x.shape[1]
    if tuple(x.shape[-nch:]) != ch:
        raise ValueError(f"x's channel dims {tuple(x.shape[-nch:])} differ from the weight's {ch}")
    _expect(state, "state", (n_seqs, *ch, width - 1))
    _expect(out, "out", x.shape)
    _expect(state_out, "state_out", (n_seqs, *ch, width - 1))
    dev, dt = x.device, x.dtype
    _need(x, "x", dt, dev)
    _need(weight, "weight", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", dt, dev)
    if state_out is None and want_state:
        state_out = torch.empty((n_seqs, *ch, width - 1), dtype=torch.float32, device=dev)
    _need(state_out, "state_out", torch.float32, dev)
    channels = 1
    for c in ch:
        channels *= c
    tokens = x.numel() // channels
    with torch.cuda.device(dev):  # the library launches on the current device
        _check(LIB.gdn_short_conv(n_seqs, seq_len, _ptr(cu_seqlens), tokens, channels, width, _dtype_code(x),
                                  _ptr(x), _ptr(weight), _ptr(state), _ptr(state_out), _ptr(out),
                                  GDN_CONV_SILU if silu else 0, _stream_handle(stream, dev)))
    return out, state_out


def launch_count() -> int:
    return int(LIB.gdn_launch_count())
