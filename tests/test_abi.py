"""The C-ABI library loads and exports every declared symbol; host-side
argument checks reject bad calls before any CUDA work (no GPU needed)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def gdn():
    from linear_attention_sequence_sm_b200 import build
    build.build()
    from linear_attention_sequence_sm_b200 import gdn as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert "gdn_chunk_forward" in names and "gdn_decode_step" in names
    assert len(names) >= 7


def test_library_exports_every_declared_symbol(gdn):
    lib = ctypes.CDLL(gdn.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(gdn.EXPORTED) == set(declared_functions())


def test_status_strings(gdn):
    for code in range(7):
        s = gdn.LIB.gdn_status_string(code).decode()
        assert s.startswith("GDN_")
    assert gdn.LIB.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"


def _shape(gdn, **kw):
    base = dict(batch=2, seq_len=64, num_seqs=2, num_qk_heads=2, num_v_heads=4, head_dim_k=128,
                head_dim_v=128, chunk_size=64, dtype=gdn.GDN_DTYPE_BF16, flags=0)
    base.update(kw)
    return gdn.Shape(**base)


def test_workspace_size(gdn):
    n = gdn.workspace_size(_shape(gdn))
    assert n >= 256 and n % 256 == 0
    big = gdn.workspace_size(_shape(gdn, batch=1, num_seqs=10000, seq_len=100000))
    assert big > n


def test_workspace_size_follows_the_path(gdn):
    """The bf16 d=128 C=64 shape runs the single tensor-core kernel by default
    (schedule-sized workspace); GDN_FLAG_SPLIT asks for the two-kernel form and
    its 16 KiB per (chunk, value head); value heads not a multiple of 4 take
    the two-kernel form by default."""
    kw = dict(batch=2, seq_len=200, num_seqs=2, num_qk_heads=2, num_v_heads=8, head_dim_k=128, head_dim_v=128,
              chunk_size=64, dtype=gdn.GDN_DTYPE_BF16)
    one = gdn.workspace_size(_shape(gdn, **kw))
    split = gdn.workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_SPLIT, **kw))
    assert split >= one + 2 * 4 * 8 * 16384  # 2 sequences x 4 chunks x 8 heads
    assert gdn.workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_ONE_KERNEL, **kw)) == one
    odd = dict(kw, num_qk_heads=1, num_v_heads=6)
    assert gdn.workspace_size(_shape(gdn, **odd)) > gdn.workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_ONE_KERNEL,
                                                                                **odd))
    # the fp32 path never takes the two-kernel form
    assert gdn.workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_SPLIT, **dict(kw, dtype=gdn.GDN_DTYPE_F32))) == one


def test_path_query_arguments(gdn):
    """The path query checks its arguments before it looks for a device (this
    host has none, so a well-formed query reports GDN_ERR_CUDA)."""
    p = ctypes.c_int32(-1)
    s = _shape(gdn)
    assert gdn.LIB.gdn_chunk_forward_path(ctypes.byref(s), ctypes.c_size_t(1 << 20), None) == \
        gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.LIB.gdn_chunk_forward_path(ctypes.byref(s), ctypes.c_size_t(0), ctypes.byref(p)) == \
        gdn.GDN_ERR_WORKSPACE_TOO_SMALL
    bad = _shape(gdn, num_v_heads=3)
    assert gdn.LIB.gdn_chunk_forward_path(ctypes.byref(bad), ctypes.c_size_t(1 << 20), ctypes.byref(p)) == \
        gdn.GDN_ERR_INVALID_ARGUMENT
    import torch
    if not torch.cuda.is_available():
        st = gdn.LIB.gdn_chunk_forward_path(ctypes.byref(s), ctypes.c_size_t(gdn.workspace_size(s)), ctypes.byref(p))
        assert st == gdn.GDN_ERR_CUDA and p.value == -1


def test_kda_workspace_size_follows_the_path(gdn):
    """The tensor-core KDA form (bf16, d = 128, C = 64) needs its 66,048 bytes
    per (chunk, value head) on top of the schedule; other shapes and
    GDN_FLAG_FORCE_SIMT need only the schedule tables."""
    kw = dict(batch=2, seq_len=200, num_seqs=2, num_qk_heads=2, num_v_heads=4, head_dim_k=128, head_dim_v=128,
              chunk_size=64, dtype=gdn.GDN_DTYPE_BF16)
    sched = gdn.workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_ONE_KERNEL, **kw))
    tc = gdn.kda_workspace_size(_shape(gdn, **kw))
    assert tc >= sched + 2 * 4 * 4 * 66048  # 2 sequences x 4 chunks x 4 value heads
    assert gdn.kda_workspace_size(_shape(gdn, flags=gdn.GDN_FLAG_FORCE_SIMT, **kw)) == sched
    assert gdn.kda_workspace_size(_shape(gdn, **dict(kw, dtype=gdn.GDN_DTYPE_F32))) == sched
    assert gdn.kda_workspace_size(_shape(gdn, **dict(kw, head_dim_k=64, head_dim_v=64))) == sched
    n = ctypes.c_size_t(0)
    bad = _shape(gdn, num_v_heads=3)
    assert gdn.LIB.gdn_kda_forward_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == gdn.GDN_ERR_INVALID_ARGUMENT


def test_noalloc_status_arguments(gdn):
    """The built-in array's status reader refuses a NULL output; on a host
    without a GPU it reports GDN_ERR_CUDA rather than reading anything."""
    assert gdn.LIB.gdn_noalloc_read_device_status(None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    import torch
    if not torch.cuda.is_available():
        st = ctypes.c_int32(-1)
        assert gdn.LIB.gdn_noalloc_read_device_status(ctypes.byref(st), None) == gdn.GDN_ERR_CUDA
        assert st.value == -1 and gdn.LIB.gdn_last_error_message().decode() != ""


def test_contradictory_path_flags_rejected(gdn):
    n = ctypes.c_size_t(0)
    s = _shape(gdn, flags=gdn.GDN_FLAG_SPLIT | gdn.GDN_FLAG_ONE_KERNEL)
    assert gdn.LIB.gdn_chunk_forward_workspace_size(ctypes.byref(s), ctypes.byref(n)) == gdn.GDN_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("kw,code", [
    (dict(num_v_heads=3), 1),          # Hv % Hk != 0
    (dict(dtype=7), 1),                # unknown dtype
    (dict(chunk_size=48), 2),          # unsupported chunk
    (dict(head_dim_k=256), 2),         # d_k > 128
    (dict(num_qk_heads=0), 1),
    (dict(seq_len=-1), 1),
])
def test_shape_rejected(gdn, kw, code):
    n = ctypes.c_size_t(0)
    st = gdn.LIB.gdn_chunk_forward_workspace_size(ctypes.byref(_shape(gdn, **kw)), ctypes.byref(n))
    assert st == code
    assert gdn.LIB.gdn_last_error_message().decode() != ""


FAKE = 0x10000000  # a 256-byte aligned address; never dereferenced: every call below fails validation first


def _call(gdn, shape, **over):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, s0=None, cu=None, o=FAKE, sf=None, ws=FAKE,
             wsb=1 << 20)
    p.update(over)
    vp = ctypes.c_void_p
    return gdn.LIB.gdn_chunk_forward(ctypes.byref(shape), vp(p["q"]), vp(p["k"]), vp(p["v"]), vp(p["g"]),
                                     vp(p["beta"]), vp(p["s0"]), vp(p["cu"]), vp(p["o"]), vp(p["sf"]),
                                     vp(p["ws"]), p["wsb"], None)


def test_null_and_misaligned_pointers(gdn):
    s = _shape(gdn)
    assert _call(gdn, s, q=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert _call(gdn, s, ws=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert _call(gdn, s, v=FAKE + 8) == gdn.GDN_ERR_MISALIGNED
    assert "v is not 16-byte aligned" in gdn.LIB.gdn_last_error_message().decode()
    assert _call(gdn, s, ws=FAKE + 16) == gdn.GDN_ERR_MISALIGNED
    assert _call(gdn, s, wsb=16) == gdn.GDN_ERR_WORKSPACE_TOO_SMALL
    # varlen needs batch 1; batched needs num_seqs == batch
    assert _call(gdn, _shape(gdn, batch=2), cu=FAKE) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert _call(gdn, _shape(gdn, num_seqs=3)) == gdn.GDN_ERR_INVALID_ARGUMENT


def test_decode_argument_checks(gdn):
    vp = ctypes.c_void_p
    f = gdn.LIB.gdn_decode_step
    args = [vp(FAKE)] * 7 + [None]
    assert f(4, 2, 3, 128, 128, 1, *args) == gdn.GDN_ERR_INVALID_ARGUMENT   # Hv % Hk
    assert f(4, 2, 4, 512, 128, 1, *args) == gdn.GDN_ERR_UNSUPPORTED        # d_k > 256
    assert f(4, 2, 4, 128, 128, 5, *args) == gdn.GDN_ERR_INVALID_ARGUMENT   # dtype
    bad = [vp(FAKE)] * 5 + [vp(FAKE + 4), vp(FAKE), None]
    assert f(4, 2, 4, 128, 128, 1, *bad) == gdn.GDN_ERR_MISALIGNED
    assert f(0, 2, 4, 128, 128, 1, *args) == gdn.GDN_OK                     # nothing to do


def test_no_device_reports_cuda_error(gdn):
    import torch
    if torch.cuda.is_available():
        pytest.skip("only meaningful without a GPU")
    assert _call(gdn, _shape(gdn)) == gdn.GDN_ERR_CUDA


def test_launch_counter_is_monotonic(gdn):
    a = gdn.launch_count()
    assert gdn.launch_count() >= a


def test_product_path_has_no_oracle_or_cpu_fallback():
    """The package and its CUDA sources never import, load or include the oracle."""
    pkg = os.path.join(ROOT, "linear_attention_sequence_sm_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"(from|import)\s+oracle|gdn_oracle|libgdn_oracle", text), fn


def _call_out(gdn, shape, osc, **over):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, o=FAKE, ws=FAKE, wsb=1 << 20)
    p.update(over)
    vp = ctypes.c_void_p
    return gdn.LIB.gdn_chunk_forward_out(ctypes.byref(shape), vp(p["q"]), vp(p["k"]), vp(p["v"]), vp(p["g"]),
                                         vp(p["beta"]), None, None, None if osc is None else ctypes.byref(osc),
                                         vp(p["o"]), None, vp(p["ws"]), p["wsb"], None)


@pytest.mark.parametrize("weight,gate,eps,flags,code", [
    (None, FAKE, 1e-6, 0, 1),            # a gate without an activation
    (None, FAKE, 1e-6, 1 | 2, 1),        # two activations
    (None, None, 1e-6, 1, 1),            # an activation without a gate
    (None, None, 0.0, 0, 1),             # eps must be > 0
    (None, None, float("nan"), 0, 1),    # and finite
    (None, None, float("inf"), 0, 1),
    (None, None, 1e-6, 16, 1),           # unknown bit
    (None, FAKE + 8, 1e-6, 1, 3),        # misaligned gate
    (FAKE + 4, None, 1e-6, 0, 3),        # misaligned weight
])
def test_output_side_rejected(gdn, weight, gate, eps, flags, code):
    osc = gdn.OutputSideC(weight, gate, eps, flags)
    assert _call_out(gdn, _shape(gdn), osc) == code
    assert gdn.LIB.gdn_last_error_message().decode() != ""
    vp = ctypes.c_void_p
    st = gdn.LIB.gdn_decode_step_out(4, 2, 4, 128, 128, 1, *([vp(FAKE)] * 6), ctypes.byref(osc), vp(FAKE), 0, None)
    assert st == code


def test_output_side_decode_dv_limit(gdn):
    vp = ctypes.c_void_p
    osc = gdn.OutputSideC(None, None, 1e-6, 0)
    st = gdn.LIB.gdn_decode_step_out(4, 2, 4, 128, 512, 1, *([vp(FAKE)] * 6), ctypes.byref(osc), vp(FAKE), 0, None)
    assert st == gdn.GDN_ERR_UNSUPPORTED


def test_output_side_valid_reaches_the_device_check(gdn):
    """A valid descriptor passes validation (no GPU here: the call then fails
    on the device query, GDN_ERR_CUDA); NULL means no output side."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("only meaningful without a GPU")
    osc = gdn.OutputSideC(FAKE, FAKE, 1e-6, 1 | 4 | 8)
    assert _call_out(gdn, _shape(gdn), osc) == gdn.GDN_ERR_CUDA
    assert _call_out(gdn, _shape(gdn), None) == gdn.GDN_ERR_CUDA


def test_decode_multi_and_commit_argument_checks(gdn):
    vp = ctypes.c_void_p
    f = gdn.LIB.gdn_decode_multi
    ptrs = [vp(FAKE)] * 8
    assert f(4, 3, 2, 4, 64, 128, 1, *ptrs, 0, None) == gdn.GDN_ERR_UNSUPPORTED   # d_k != 128
    assert f(4, 17, 2, 4, 128, 128, 1, *ptrs, 0, None) == gdn.GDN_ERR_UNSUPPORTED  # more than 16 tokens
    assert f(4, 0, 2, 4, 128, 128, 1, *ptrs, 0, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert f(4, 3, 2, 3, 128, 128, 1, *ptrs, 0, None) == gdn.GDN_ERR_INVALID_ARGUMENT  # Hv % Hk
    assert f(4, 3, 2, 4, 128, 128, 1, *ptrs, 8, None) == gdn.GDN_ERR_INVALID_ARGUMENT  # unknown flag
    bad = [vp(FAKE)] * 6 + [vp(FAKE + 4), vp(FAKE)]
    assert f(4, 3, 2, 4, 128, 128, 1, *bad, 0, None) == gdn.GDN_ERR_MISALIGNED
    nul = [vp(FAKE)] * 6 + [None, vp(FAKE)]
    assert f(4, 3, 2, 4, 128, 128, 1, *nul, 0, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert f(0, 3, 2, 4, 128, 128, 1, *ptrs, 0, None) == gdn.GDN_OK
    c = gdn.LIB.gdn_decode_commit
    assert c(4, 3, 4, 128, 128, None, vp(FAKE), vp(FAKE), None, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert c(4, 3, 4, 128, 128, vp(FAKE + 8), vp(FAKE), vp(FAKE), None, None) == gdn.GDN_ERR_MISALIGNED
    assert c(4, 3, 4, 3, 3, vp(FAKE), vp(FAKE), vp(FAKE), None, None) == gdn.GDN_ERR_UNSUPPORTED
    assert c(0, 3, 4, 128, 128, None, None, None, None, None) == gdn.GDN_OK


def test_backward_workspace_size_follows_the_path(gdn):
    """bf16 with d_k = d_v = 128 sizes the tensor-core backward: the schedule
    and chunk_base, then 212,992 + 2 x 65,536 bytes per (chunk, value head)
    slot; GDN_FLAG_FORCE_SIMT, fp32 or other head sizes size the single-kernel
    form; the forward-path flags are refused by the backward."""
    n = ctypes.c_size_t(0)
    def size(**kw):
        assert gdn.LIB.gdn_chunk_backward_workspace_size(ctypes.byref(_shape(gdn, **kw)), ctypes.byref(n)) == gdn.GDN_OK
        return n.value
    # 2 sequences of 200 tokens, 4 value heads: at most (400 + 63 * 2) // 64 = 8 chunks; the tables
    # (header, order, start, len: 1024 bytes; chunk_base) end at 2048 after rounding to 1 KiB
    tc = size(batch=2, seq_len=200, num_seqs=2)
    assert tc == 2048 + 8 * 4 * (212992 + 2 * 65536)
    simt = size(batch=2, seq_len=200, num_seqs=2, flags=gdn.GDN_FLAG_FORCE_SIMT)
    assert simt != tc
    assert size(batch=2, seq_len=200, num_seqs=2, dtype=gdn.GDN_DTYPE_F32) == simt
    assert size(batch=2, seq_len=200, num_seqs=2, head_dim_k=64, head_dim_v=64) not in (tc, simt)
    # the tensor-core size grows with the chunks, one slot per (chunk, value head)
    assert size(batch=2, seq_len=264, num_seqs=2) - tc == 2 * 4 * (212992 + 2 * 65536)
    vp = ctypes.c_void_p
    for flag in (gdn.GDN_FLAG_ONE_KERNEL, gdn.GDN_FLAG_SPLIT):
        s = _shape(gdn, flags=flag)
        st = gdn.LIB.gdn_chunk_backward(ctypes.byref(s), *(vp(FAKE) for _ in range(5)), None, None, vp(FAKE), None,
                                        *(vp(FAKE) for _ in range(5)), None, vp(FAKE), ctypes.c_size_t(1 << 40), None)
        assert st == gdn.GDN_ERR_UNSUPPORTED


def test_backward_and_kda_argument_checks(gdn):
    """Refused before any device work: input-side flags on the backward,
    NULL gradient outputs, a short workspace, misalignment; KDA with d_k > 128."""
    vp = ctypes.c_void_p
    s = _shape(gdn, chunk_size=32)
    n = ctypes.c_size_t(0)
    assert gdn.LIB.gdn_chunk_backward_workspace_size(ctypes.byref(s), ctypes.byref(n)) == gdn.GDN_OK
    assert n.value > gdn.workspace_size(s)  # the chunk checkpoints come on top of the schedule

    def bwd(shape, **over):
        p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, s0=None, cu=None, do=FAKE, dsf=None, dq=FAKE, dk=FAKE,
                 dv=FAKE, dg=FAKE, db=FAKE, ds0=None, ws=FAKE, wsb=n.value)
        p.update(over)
        return gdn.LIB.gdn_chunk_backward(ctypes.byref(shape), *(vp(p[k]) for k in (
            "q", "k", "v", "g", "beta", "s0", "cu", "do", "dsf", "dq", "dk", "dv", "dg", "db", "ds0", "ws")),
            p["wsb"], None)

    assert bwd(_shape(gdn, chunk_size=32, flags=2)) == gdn.GDN_ERR_UNSUPPORTED
    assert bwd(s, dq=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert bwd(s, wsb=1024) == gdn.GDN_ERR_WORKSPACE_TOO_SMALL
    assert bwd(s, dv=FAKE + 4) == gdn.GDN_ERR_MISALIGNED
    assert bwd(_shape(gdn, chunk_size=32, head_dim_k=256)) == gdn.GDN_ERR_UNSUPPORTED
    ks = _shape(gdn, head_dim_k=160)
    st = gdn.LIB.gdn_kda_forward(ctypes.byref(ks), *([vp(FAKE)] * 5), None, None, None, vp(FAKE), None, vp(FAKE),
                                 1 << 20, None)
    assert st == gdn.GDN_ERR_UNSUPPORTED
    st = gdn.LIB.gdn_kda_decode_step(4, 2, 4, 512, 128, 1, *([vp(FAKE)] * 6), None, vp(FAKE), 0, None)
    assert st == gdn.GDN_ERR_UNSUPPORTED


def test_short_conv_argument_checks(gdn):
    """Refused before any device work: widths outside 1..8, channels not a
    multiple of 4, a token count that the batched layout does not give,
    aliased outputs, misalignment; no sequences is a no-op; a valid call
    reaches the device check."""
    vp = ctypes.c_void_p
    f = gdn.LIB.gdn_short_conv

    def conv(n=2, seq_len=5, cu=None, tokens=10, ch=256, w=4, dt=1, x=FAKE, wt=FAKE, si=None, so=None, y=FAKE + 4096,
             flags=1):
        return f(n, seq_len, None if cu is None else vp(cu), tokens, ch, w, dt, vp(x) if x else None,
                 vp(wt) if wt else None, vp(si) if si else None, vp(so) if so else None, vp(y) if y else None,
                 flags, None)

    assert conv(w=0) == gdn.GDN_ERR_UNSUPPORTED and conv(w=9) == gdn.GDN_ERR_UNSUPPORTED
    assert conv(ch=6) == gdn.GDN_ERR_UNSUPPORTED
    assert conv(tokens=11) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert conv(flags=2) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert conv(dt=7) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert conv(y=FAKE) == gdn.GDN_ERR_INVALID_ARGUMENT  # y aliases x
    assert conv(si=FAKE + 8192, so=FAKE + 8192) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert conv(wt=None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert conv(x=FAKE + 4) == gdn.GDN_ERR_MISALIGNED
    assert conv(n=0, tokens=0) == gdn.GDN_OK
    assert conv(n=0, tokens=4, cu=FAKE) == gdn.GDN_ERR_INVALID_ARGUMENT
    import torch
    if not torch.cuda.is_available():  # with a GPU this call would launch on the fake pointers
        assert conv() == gdn.GDN_ERR_CUDA  # everything valid: the next step needs a GPU


def test_header_is_plain_c(tmp_path):
    """include/gdn.h compiles as pedantic C99 (plain pointers and sizes, no
    C++ or torch types in the ABI)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "gdn.h"\nint main(void) { gdn_output_side_t o = {0}; (void)o; '
                   'return (int)sizeof(gdn_shape_t); }\n')
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
