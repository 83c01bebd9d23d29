"""The index walk of the short-convolution kernel (csrc/gdn_conv.cu), written
out in Python thread by thread and run on CPU against the fp64 oracle.

The kernel gives each thread a segment of kConvSeg consecutive tokens of the
packed layout and a group of channels.  A segment may start inside a
sequence, span several short ones, or include empty ones; the thread finds
the sequence of its first token by binary search over cu_seqlens, fills its
W-1 token history from the inputs before the segment (or from the
sequence's conv state, or zeros, before the sequence's first token), and
walks its tokens, resetting the history at each sequence start and writing
the conv state after each sequence's last token.  Empty sequences get their
state passed through by a second kernel.  This file checks that walk; the
GPU parity test checks the kernel itself."""
import numpy as np
import pytest

SEG = 64  # tokens per thread segment, as kConvSeg in the kernel


def upper_bound(cu, t):
    """Index of the first entry of cu greater than t (the kernel's binary search)."""
    lo, hi = 0, len(cu)
    while lo < hi:
        mid = (lo + hi) // 2
        if cu[mid] <= t:
            lo = mid + 1
        else:
            hi = mid
    return lo


def walk(x, w, cu, state_in, silu, seg=SEG):
    """The kernels' arithmetic and indexing, per (segment, channel) thread,
    in fp64 so that only the walk, not the rounding, is under test."""
    T, C = x.shape
    W = w.shape[1]
    H = W - 1
    N = len(cu) - 1
    y = np.full((T, C), np.nan)
    s_out = np.full((N, C, H), np.nan)
    for c in range(C):
        for t0 in range(0, T, seg):
            t1 = min(t0 + seg, T)
            n = upper_bound(cu, t0) - 1  # cu[n] <= t0 < cu[n + 1]
            hist = []
            for i in range(H):
                u = t0 - H + i
                if u >= cu[n]:
                    hist.append(x[u, c])
                else:
                    hist.append(state_in[n, c, H - (cu[n] - u)] if state_in is not None else 0.0)
            for t in range(t0, t1):
                while t >= cu[n + 1]:
                    n += 1
                    hist = [state_in[n, c, i] if state_in is not None else 0.0 for i in range(H)]
                acc = w[c, H] * x[t, c]
                for j in range(H):
                    acc += w[c, j] * hist[j]
                y[t, c] = acc / (1.0 + np.exp(-acc)) if silu else acc
                hist = hist[1:] + [x[t, c]]
                if t == cu[n + 1] - 1:
                    s_out[n, c] = hist
    # second kernel: empty sequences pass their state through
    for n in range(N):
        if cu[n + 1] == cu[n]:
            s_out[n] = state_in[n] if state_in is not None else 0.0
    return y, s_out


@pytest.mark.parametrize("case", range(12))
def test_walk_matches_oracle(oracle_mod, case):
    rng = np.random.default_rng(900 + case)
    W = [1, 2, 3, 4, 4, 4, 5, 8, 4, 4, 2, 4][case]
    seg = [64, 64, 64, 64, 5, 3, 7, 4, 1, 2, 64, 9][case]
    n = int(rng.integers(1, 9))
    lens = [int(v) for v in rng.integers(0, 3 * seg + 4, size=n)]
    if case % 3 == 0:
        lens[rng.integers(0, n)] = 0
    lens.append(int(rng.integers(1, 5)))  # at least one token in all
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    C = 3
    x = rng.standard_normal((int(cu[-1]), C))
    w = rng.standard_normal((C, W))
    st = rng.standard_normal((len(lens), C, W - 1)) if case % 2 else None
    for silu in (False, True):
        y, s = walk(x, w, cu, st, silu, seg)
        y_ref, s_ref = oracle_mod.short_conv(x, w, cu_seqlens=cu, state=st, silu=silu)
        assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-14)
        assert np.allclose(s, s_ref, rtol=0, atol=0)
