"""Plant mistakes in a copy of the oracle and check that the pins catch each.

Every mutant is a plausible slip (a dropped term, a wrong sign, a wrong
index or head mapping, an ignored state, a misplaced decay).  The mutated
copy is compiled into a temporary library; the pins of
``test_oracle_pins.py`` run against it; at least one must fail.  The real
oracle source is never modified.
"""
import os

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "gdn_oracle.c")

# (name, text to find, replacement); only the first occurrence is replaced,
# which for the shared idioms is the one inside the token recurrence.
MUTANTS = [
    ("erase term without alpha",
     "const double ui = beta * (vt[i] - alpha * pk[i]);", "const double ui = beta * (vt[i] - pk[i]);"),
    ("beta dropped",
     "const double ui = beta * (vt[i] - alpha * pk[i]);", "const double ui = (vt[i] - alpha * pk[i]);"),
    ("write with wrong sign",
     "S[i * dk + j] = alpha * S[i * dk + j] + ui * kt[j];", "S[i * dk + j] = alpha * S[i * dk + j] - ui * kt[j];"),
    ("decay applied to the write too",
     "S[i * dk + j] = alpha * S[i * dk + j] + ui * kt[j];",
     "S[i * dk + j] = alpha * (S[i * dk + j] + ui * kt[j]);"),
    ("read-out with k instead of q",
     "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];",
     "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kt[j];"),
    ("modulo head mapping",
     "const int hq = h / (p->hv / p->hk);", "const int hq = h % p->hk;"),
    ("initial state ignored",
     "if (p->s0) memcpy(S, p->s0 + unit", "if (0) memcpy(S, p->s0 + unit"),
    ("gate sign flipped",
     "const double alpha = exp(p->g[t * p->hv + h]);", "const double alpha = exp(-p->g[t * p->hv + h]);"),
    ("chunk mask without its diagonal",
     "for (int j = 0; j <= r; ++j) {", "for (int j = 0; j < r; ++j) {"),
    ("triangular solve with wrong sign",
     "x -= A[r * L + j] * T[j * L + c];", "x += A[r * L + j] * T[j * L + c];"),
    ("W without the cumulative decay",
     "acc += T[r * L + j] * p->beta[(c0 + j) * p->hv + h] * exp(G[j]) * K[j * dk + x];",
     "acc += T[r * L + j] * p->beta[(c0 + j) * p->hv + h] * K[j * dk + x];"),
    ("carried state not decayed",
     "S[i * dk + x] = exp(gl) * S[i * dk + x] + acc;", "S[i * dk + x] = S[i * dk + x] + acc;"),
    ("inter-chunk output term without gamma",
     "ot[i] = exp(G[r]) * inter + intra;", "ot[i] = inter + intra;"),
    ("q left unnormalised",
     "double *xs[2] = {q, k};", "double *xs[2] = {k, k};"),
    ("sigmoid used as the log-decay",
     "g[r] = a >= 0.0 ? -log1p(exp(-a)) : a - log1p(exp(a));", "g[r] = 1.0 / (1.0 + exp(-a));"),
    ("log-decay of the negated logit",
     "g[r] = a >= 0.0 ? -log1p(exp(-a)) : a - log1p(exp(a));", "g[r] = a >= 0.0 ? -a - log1p(exp(-a)) : -log1p(exp(a));"),
    ("RMS over the sum of squares, not the mean",
     "    ms /= dv;\n", "\n"),
    ("eps outside the root",
     "const double inv_rms = 1.0 / sqrt(ms + eps);", "const double inv_rms = 1.0 / (sqrt(ms) + eps);"),
    ("SiLU gate without its z factor",
     "gate = z[row + i] / (1.0 + exp(-z[row + i]));", "gate = 1.0 / (1.0 + exp(-z[row + i]));"),
    ("zero-centred scale without its 1",
     "if (out_flags & 4u) s = 1.0 + (wr ? wr[i] : 0.0);", "if (out_flags & 4u) s = (wr ? wr[i] : 0.0);"),
    ("per-head scale rows ignored",
     "const double *wr = w ? w + ((out_flags & 8u) ? (int64_t)h * dv : 0) : NULL;",
     "const double *wr = w;"),
    ("KDA prediction from the undecayed row",
     "pred += sd[j] * kt[j];", "pred += S[i * dk + j] * kt[j];"),
    ("KDA decay of one channel for all",
     "for (int j = 0; j < dk; ++j) alpha[j] = exp(gt[j]);", "for (int j = 0; j < dk; ++j) alpha[j] = exp(gt[0]);"),
    ("KDA write without beta",
     "const double ui = beta * (vt[i] - pred);", "const double ui = (vt[i] - pred);"),
    ("KDA chunk A with the decay transposed",
     "a += KDA_K(r, c) * KDA_K(j, c) * exp(G[r * dk + c] - G[j * dk + c]);",
     "a += KDA_K(r, c) * KDA_K(j, c) * exp(G[j * dk + c] - G[r * dk + c]);"),
    ("KDA chunk output without the start-state decay",
     "acc += S[i * dk + c] * KDA_Q(r, c) * exp(G[r * dk + c]);", "acc += S[i * dk + c] * KDA_Q(r, c);"),
    ("KDA chunk end state without the decay of the writes",
     "acc += U[j * dv + i] * KDA_K(j, c) * exp(Gl[c] - G[j * dk + c]);", "acc += U[j * dv + i] * KDA_K(j, c);"),
    ("backward: decay gradient without alpha",
     "gr->dg[tt * p->hv + h] = alpha * dalpha;", "gr->dg[tt * p->hv + h] = dalpha;"),
    ("backward: carried state gradient not decayed",
     "for (size_t e = 0; e < ssz; ++e) dS[e] = alpha * dsp[e];", "for (size_t e = 0; e < ssz; ++e) dS[e] = dsp[e];"),
    ("backward: key gradient without the write term",
     "dkt[j] += u[i] * dS[i * dk + j] + dpi * alpha * Sp[i * dk + j];", "dkt[j] += dpi * alpha * Sp[i * dk + j];"),
    ("backward chunked: inverse gradient with the wrong sign",
     "dA[r * L + j] = -acc;", "dA[r * L + j] = acc;"),
    ("backward chunked: end-state decay gradient dropped",
     "dG[L - 1] += dgL * gL;", "dG[L - 1] += 0.0 * dgL;"),
    ("recurrence stops one token early",
     "for (int64_t t = p->cu_seqlens[n]; t < p->cu_seqlens[n + 1]; ++t) {",
     "for (int64_t t = p->cu_seqlens[n]; t < p->cu_seqlens[n + 1] - 1; ++t) {"),
    ("every sequence starts from the first sequence's state",
     "if (p->s0) memcpy(S, p->s0 + unit * (int64_t)dv * dk,", "if (p->s0) memcpy(S, p->s0 + (int64_t)h * dv * dk,"),
    ("chunk grid on the packed token index, not the sequence start",
     "for (int64_t c0 = t_begin; c0 < t_end; c0 += C, ++chunk_idx) {",
     "for (int64_t c0 = t_begin - t_begin % C; c0 < t_end; c0 += C, ++chunk_idx) {"),
    ("backward: reverse walk stops before the first token",
     "for (int64_t t = T - 1; t >= 0; --t) {", "for (int64_t t = T - 1; t >= 1; --t) {"),
    ("conv taps reversed",
     "acc += w[(int64_t)c * width + j] * CONV_IN(t - hist + j);",
     "acc += w[(int64_t)c * width + (width - 1 - j)] * CONV_IN(t - hist + j);"),
    ("conv reads across the sequence start",
     "#define CONV_IN(u) ((u) >= s ?", "#define CONV_IN(u) ((u) >= 0 ?"),
    ("conv state ignored",
     "(st ? st[hist - (s - (u))] : 0.0)", "(0.0)"),
    ("conv activation a sigmoid, not SiLU",
     "y[t * channels + c] = silu ? acc / (1.0 + exp(-acc)) : acc;",
     "y[t * channels + c] = silu ? 1.0 / (1.0 + exp(-acc)) : acc;"),
    ("A built with Gamma transposed",
     "a = p->beta[(c0 + r) * p->hv + h] * exp(G[r] - G[j]) * kk;",
     "a = p->beta[(c0 + r) * p->hv + h] * exp(G[j] - G[r]) * kk;"),
]


class _Bound:
    """The oracle module's API bound to a given (mutant) library."""

    def __init__(self, lib):
        self.lib = lib

    def recurrent(self, *a, **kw):
        return oracle.recurrent(*a, lib=self.lib, **kw)

    def chunkwise(self, *a, **kw):
        return oracle.chunkwise(*a, lib=self.lib, **kw)

    def delta_error_form(self, *a, **kw):
        return oracle.delta_error_form(*a, lib=self.lib, **kw)

    def decode_step(self, *a, **kw):
        return oracle.decode_step(*a, lib=self.lib, **kw)

    def prepare_inputs(self, *a, **kw):
        return oracle.prepare_inputs(*a, lib=self.lib, **kw)

    def output_side(self, *a, **kw):
        return oracle.output_side(*a, lib=self.lib, **kw)

    def backward(self, *a, **kw):
        return oracle.backward(*a, lib=self.lib, **kw)

    def kda_recurrent(self, *a, **kw):
        return oracle.kda_recurrent(*a, lib=self.lib, **kw)

    def kda_chunkwise(self, *a, **kw):
        return oracle.kda_chunkwise(*a, lib=self.lib, **kw)

    def short_conv(self, *a, **kw):
        return oracle.short_conv(*a, lib=self.lib, **kw)


def _pin_calls(m):
    return [
        lambda: pins.test_handworked_example(m),
        lambda: pins.test_one_token_and_head_mapping(m),
        lambda: pins.test_g_zero_is_delta_rule(m, True),
        lambda: pins.test_beta_zero_decay_only(m),
        lambda: pins.test_exact_recall_orthonormal_keys(m),
        lambda: pins.test_alpha_zero_clears_state(m),
        lambda: pins.test_brute_force_explicit_matrices(m),
        lambda: pins.test_chunkwise_equals_recurrent(m, 4, True),
        lambda: pins.test_chunkwise_equals_recurrent(m, 16, False),
        lambda: pins.test_continuation(m, 13),
        lambda: pins.test_varlen_equals_per_sequence(m),
        lambda: pins.test_prepare_closed_forms(m),
        lambda: pins.test_prepared_one_token_closed_form(m),
        lambda: pins.test_output_side_handworked(m),
        lambda: pins.test_output_side_invariants(m),
        lambda: pins.test_kda_scalar_decay_is_gated_delta_rule(m),
        lambda: pins.test_kda_brute_force_explicit_matrices(m),
        lambda: pins.test_kda_beta_zero_is_channel_decay(m),
        lambda: pins.test_kda_one_token(m),
        lambda: pins.test_kda_chunkwise_equals_recurrent(m, 4),
        lambda: pins.test_backward_matches_finite_differences(m),
        lambda: pins.test_backward_chunkwise_equals_token_recurrence(m, 4),
        lambda: pins.test_short_conv_identity_and_shift(m),
        lambda: pins.test_short_conv_equals_numpy_correlate(m),
        lambda: pins.test_short_conv_continuation(m),
    ]


def _caught(m):
    failures = 0
    for call in _pin_calls(m):
        try:
            with np.errstate(all="ignore"):
                call()
        except AssertionError:
            failures += 1
    return failures


def test_unmutated_copy_passes(tmp_path):
    src = open(SRC).read()
    p = tmp_path / "copy.c"
    p.write_text(src)
    lib = oracle.load(oracle.build(force=True, src=str(p), out=str(tmp_path / "libcopy.so")))
    assert _caught(_Bound(lib)) == 0


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, find, repl):
    src = open(SRC).read()
    assert find in src, f"mutation anchor missing: {find}"
    p = tmp_path / "mutant.c"
    p.write_text(src.replace(find, repl, 1))
    lib = oracle.load(oracle.build(force=True, src=str(p), out=str(tmp_path / "libmutant.so")))
    assert _caught(_Bound(lib)) > 0, f"no pin caught the mutant: {name}"
