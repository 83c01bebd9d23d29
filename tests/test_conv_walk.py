"""The index walk of the short-convolution kernels (csrc/gdn_conv.cu), written
out in Python thread by thread and run on CPU against the fp64 oracle.

The convolution kernel gives each thread kConvTok consecutive tokens of the
packed layout and a group of channels.  The thread loads the input rows from
W-1 before its first token to its last token (zeros outside the tensor),
finds the sequence of its first token by binary search over cu_seqlens, and
for each of its tokens steps on to the token's sequence; a tap before the
sequence's first token reads the sequence's conv state (or zero).  The thread
holding a sequence's last token writes that sequence's last W-1 inputs,
reaching into the incoming state when the sequence is shorter; a second
kernel passes the state of empty sequences through.  This file checks that
walk with several tokens-per-thread counts; the GPU parity test checks the
kernels themselves."""
import numpy as np
import pytest

TOK = 8  # tokens per thread, as kConvTok in the kernel


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


def walk(x, w, cu, state_in, silu, tok=TOK):
    """The kernels' arithmetic and indexing, per (token group, channel) thread,
    in fp64 so that only the walk, not the rounding, is under test."""
    T, C = x.shape
    W = w.shape[1]
    H = W - 1
    N = len(cu) - 1
    y = np.full((T, C), np.nan)
    s_out = np.full((N, C, H), np.nan)

    def from_state(n, c, start, u):
        si = H - (start - u)  # oldest first in the conv state
        return state_in[n, c, si] if (state_in is not None and 0 <= si < H) else 0.0

    for c in range(C):
        for t0 in range(0, T, tok):
            rows = {u: (x[u, c] if 0 <= u < T else 0.0) for u in range(t0 - H, t0 + tok)}
            n = min(max(upper_bound(cu, t0) - 1, 0), N - 1)
            start, nxt = cu[n], cu[n + 1]
            for t in range(t0, min(t0 + tok, T)):
                while t >= nxt and n < N - 1:
                    n += 1
                    start, nxt = nxt, cu[n + 1]
                acc = 0.0
                for j in range(W):
                    u = t - H + j
                    acc += w[c, j] * (rows[u] if u >= start else from_state(n, c, start, u))
                y[t, c] = acc / (1.0 + np.exp(-acc)) if silu else acc
                if t == nxt - 1:  # the sequence's last token: its conv state
                    for i in range(H):
                        u = t - H + 1 + i
                        s_out[n, c, i] = rows[u] if u >= start else from_state(n, c, start, u)
    # the second kernel: empty sequences pass their state through
    for n in range(N):
        if cu[n + 1] == cu[n]:
            s_out[n] = state_in[n] if state_in is not None else 0.0
    return y, s_out


@pytest.mark.parametrize("case", range(12))
def test_walk_matches_oracle(oracle_mod, case):
    rng = np.random.default_rng(900 + case)
    W = [1, 2, 3, 4, 4, 4, 5, 8, 4, 4, 2, 4][case]
    seg = [8, 8, 8, 8, 5, 3, 7, 4, 1, 2, 64, 9][case]
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
