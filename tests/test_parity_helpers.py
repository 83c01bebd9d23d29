"""CPU checks of the parity helpers that the GPU tests rely on: the
all-units comparison reproduces an exact match as zero error, and its
per-chunk metric exposes one wrong chunk that the per-slice metric hides."""
import numpy as np
import torch

from linear_attention_sequence_sm_b200 import inputs as I
from parity import full_prefill_errors, oracle_prefill


def _exact(inp):
    o_ref, s_ref = oracle_prefill(inp)
    return torch.tensor(np.asarray(o_ref)), torch.tensor(np.asarray(s_ref))


def test_all_units_exact_match_batched():
    w = I.custom("helper_b", batch=2, seq_len=1024, hk=2, hv=4, d=16, chunk=64, dtype="f32", seed=7,
                 s0_std=0.02)
    inp = I.make_prefill_inputs(w)
    o, sf = _exact(inp)
    r = full_prefill_errors(inp, o, sf, threads=2)
    assert r["units"] == 2 * 4
    assert r["o_slice"] == 0.0 and r["o_chunk"] == 0.0 and r["state"] == 0.0


def test_chunk_metric_catches_one_wrong_chunk():
    """5% error on one 64-token chunk of a 1024-token slice: about 1.3% over
    the slice (under the 2e-2 bar) but 5% over the chunk."""
    w = I.custom("helper_c", batch=2, seq_len=1024, hk=1, hv=2, d=16, chunk=64, dtype="f32", seed=8)
    inp = I.make_prefill_inputs(w)
    o, sf = _exact(inp)
    o[1, 320:384, 1] *= 1.05
    r = full_prefill_errors(inp, o, sf)
    assert r["o_slice"] < 2e-2 < r["o_chunk"], r
    assert abs(r["o_chunk"] - 0.05) < 1e-9


def test_all_units_varlen_with_empty_and_ragged():
    """Packed sequences (an empty one, ragged tails): the last chunk of each
    sequence is its own segment, and a wrong final state is seen."""
    w = I.custom("helper_v", 1, 0, 1, 3, 16, 64, "f32", seed=9, s0_std=0.02, seq_lens=[70, 0, 129, 1])
    inp = I.make_prefill_inputs(w)
    o, sf = _exact(inp)
    r = full_prefill_errors(inp, o, sf)
    assert r["units"] == 4 * 3 and r["o_chunk"] == 0.0
    o2 = o.clone()
    o2[0, 70 + 128, 2] += 1.0      # the one-token last chunk of the third sequence
    sf2 = sf.clone()
    sf2[1, 0] *= 2.0               # the empty sequence's state (= its initial state)
    r = full_prefill_errors(inp, o2, sf2)
    assert r["o_chunk"] > 0.5 and abs(r["state"] - 1.0) < 1e-12, r
