"""The binding's shape checks (CPU).  The C ABI takes bare pointers and
derives every extent from q and v, so the binding must reject a tensor of
any other shape before a kernel could read or write past it.  These checks
run before the device checks, so CPU tensors exercise them: a mis-shaped
argument raises ValueError naming it; correctly shaped CPU tensors get past
them and stop at the device check."""
import pytest
import torch

B, T, HK, HV, DK, DV = 2, 10, 1, 2, 16, 8


def prefill(**over):
    x = {"q": torch.zeros(B, T, HK, DK), "k": torch.zeros(B, T, HK, DK), "v": torch.zeros(B, T, HV, DV),
         "g": torch.zeros(B, T, HV), "beta": torch.zeros(B, T, HV), "initial_state": None, "cu_seqlens": None}
    x.update(over)
    return x


def call_forward(fn, x, **kw):
    return fn(x["q"], x["k"], x["v"], x["g"], x["beta"], initial_state=x["initial_state"],
              cu_seqlens=x["cu_seqlens"], **kw)


def device_error(excinfo):
    return "CUDA tensor" in str(excinfo.value)


@pytest.mark.parametrize("name", ["chunk_forward", "chunk_forward_noalloc"])
def test_prefill_good_shapes_reach_the_device_check(name):
    from linear_attention_sequence_sm_b200 import gdn
    with pytest.raises(ValueError) as e:
        call_forward(getattr(gdn, name), prefill(initial_state=torch.zeros(B, HV, DV, DK)))
    assert device_error(e)


@pytest.mark.parametrize("over,what", [
    ({"k": torch.zeros(B, T, HK, DK + 1)}, "k"),
    ({"v": torch.zeros(B, T + 1, HV, DV)}, "v"),
    ({"v": torch.zeros(T, HV, DV)}, "v"),
    ({"g": torch.zeros(B, T)}, "g"),
    ({"g": torch.zeros(B, T, HV, DK)}, "g"),
    ({"beta": torch.zeros(B, T, HV + 1)}, "beta"),
    ({"initial_state": torch.zeros(B, HV, DK, DV)}, "initial_state"),  # d_v and d_k swapped
    ({"initial_state": torch.zeros(B + 1, HV, DV, DK)}, "initial_state"),
    ({"q": torch.zeros(T, HK, DK), "k": torch.zeros(T, HK, DK)}, "batched q"),
])
def test_prefill_rejects_mis_shaped_inputs(over, what):
    from linear_attention_sequence_sm_b200 import gdn
    with pytest.raises(ValueError) as e:
        call_forward(gdn.chunk_forward, prefill(**over))
    assert what in str(e.value) and not device_error(e)


def test_prefill_rejects_mis_shaped_outputs():
    from linear_attention_sequence_sm_b200 import gdn
    with pytest.raises(ValueError, match="out must have shape"):
        call_forward(gdn.chunk_forward, prefill(), out=torch.zeros(B, T, HV, DV + 1))
    with pytest.raises(ValueError, match="final_state must have shape"):
        call_forward(gdn.chunk_forward, prefill(), final_state=torch.zeros(B, HV, DV, DV))


def test_varlen_layouts():
    """Packed sequences: q is [T, Hk, d_k] or [1, T, Hk, d_k]; the states
    follow the length of cu_seqlens, not the batch."""
    from linear_attention_sequence_sm_b200 import gdn
    cu = torch.tensor([0, 4, 4, T], dtype=torch.int32)
    packed = prefill(q=torch.zeros(1, T, HK, DK), k=torch.zeros(1, T, HK, DK), v=torch.zeros(1, T, HV, DV),
                     g=torch.zeros(1, T, HV), beta=torch.zeros(1, T, HV), cu_seqlens=cu,
                     initial_state=torch.zeros(3, HV, DV, DK))
    with pytest.raises(ValueError) as e:
        call_forward(gdn.chunk_forward, packed)
    assert device_error(e)
    flat = dict(packed, q=packed["q"][0], k=packed["k"][0], v=packed["v"][0], g=packed["g"][0],
                beta=packed["beta"][0])
    with pytest.raises(ValueError) as e:
        call_forward(gdn.chunk_forward, flat)
    assert device_error(e)
    with pytest.raises(ValueError, match="initial_state"):
        call_forward(gdn.chunk_forward, dict(packed, initial_state=torch.zeros(1, HV, DV, DK)))
    with pytest.raises(ValueError, match="with cu_seqlens q"):
        call_forward(gdn.chunk_forward, prefill(cu_seqlens=cu))  # batch of 2 with cu_seqlens
    with pytest.raises(ValueError, match="cu_seqlens must be"):
        call_forward(gdn.chunk_forward, dict(packed, cu_seqlens=cu[None]))


def test_kda_gate_shape():
    from linear_attention_sequence_sm_b200 import gdn
    with pytest.raises(ValueError) as e:
        call_forward(gdn.kda_forward, prefill(g=torch.zeros(B, T, HV, DK)))
    assert device_error(e)
    with pytest.raises(ValueError, match="g must have shape"):
        call_forward(gdn.kda_forward, prefill())  # one decay per head is not KDA's


def test_backward_gradient_inputs():
    from linear_attention_sequence_sm_b200 import gdn
    x = prefill()
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"])
    with pytest.raises(ValueError) as e:
        gdn.chunk_backward(*args, torch.zeros(B, T, HV, DV), d_final_state=torch.zeros(B, HV, DV, DK))
    assert device_error(e)
    with pytest.raises(ValueError, match="d_o must have shape"):
        gdn.chunk_backward(*args, torch.zeros(B, T - 1, HV, DV))
    with pytest.raises(ValueError, match="d_final_state must have shape"):
        gdn.chunk_backward(*args, torch.zeros(B, T, HV, DV), d_final_state=torch.zeros(B, HV, DK, DV))


N = 3


def decode(**over):
    x = {"q": torch.zeros(N, HK, DK), "k": torch.zeros(N, HK, DK), "v": torch.zeros(N, HV, DV),
         "g": torch.zeros(N, HV), "beta": torch.zeros(N, HV), "state": torch.zeros(N, HV, DV, DK)}
    x.update(over)
    return x


def call_decode(fn, x, **kw):
    return fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"], **kw)


def test_decode_shapes():
    from linear_attention_sequence_sm_b200 import gdn
    with pytest.raises(ValueError) as e:
        call_decode(gdn.decode_step, decode())
    assert device_error(e)
    for over, what in (({"v": torch.zeros(N + 1, HV, DV)}, "v"), ({"g": torch.zeros(N, HV, 1)}, "g"),
                       ({"beta": torch.zeros(N)}, "beta"), ({"state": torch.zeros(N, HV, DK, DV)}, "state"),
                       ({"q": torch.zeros(1, N, HK, DK)}, "q")):
        with pytest.raises(ValueError) as e:
            call_decode(gdn.decode_step, decode(**over))
        assert what in str(e.value) and not device_error(e), (what, str(e.value))
    with pytest.raises(ValueError, match="out must have shape"):
        call_decode(gdn.decode_step, decode(), out=torch.zeros(N, HV, DV + 1))
    with pytest.raises(ValueError) as e:
        call_decode(gdn.kda_decode_step, decode(g=torch.zeros(N, HV, DK)))
    assert device_error(e)
    with pytest.raises(ValueError, match="g must have shape"):
        call_decode(gdn.kda_decode_step, decode())


def test_multi_token_decode_and_commit_shapes():
    from linear_attention_sequence_sm_b200 import gdn
    K = 3
    q, v = torch.zeros(N, K, HK, 128), torch.zeros(N, K, HV, DV)
    g, b, st = torch.zeros(N, K, HV), torch.zeros(N, K, HV), torch.zeros(N, HV, DV, 128)
    with pytest.raises(ValueError) as e:
        gdn.decode_multi(q, q, v, g, b, st)
    assert device_error(e)
    with pytest.raises(ValueError, match="g must have shape"):
        gdn.decode_multi(q, q, v, torch.zeros(N, HV), b, st)
    with pytest.raises(ValueError, match="v must be"):
        gdn.decode_multi(q, q, torch.zeros(N, K + 1, HV, DV), g, b, st)
    with pytest.raises(ValueError, match="snapshots must have shape"):
        gdn.decode_multi(q, q, v, g, b, st, snapshots=torch.zeros(N, K, HV, DV, 64))
    snaps = torch.zeros(N, K, HV, DV, 128)
    acc = torch.zeros(N, dtype=torch.int32)
    with pytest.raises(ValueError) as e:
        gdn.decode_commit(snaps, acc, st)
    assert device_error(e)
    with pytest.raises(ValueError, match="accepted must have shape"):
        gdn.decode_commit(snaps, torch.zeros(N + 1, dtype=torch.int32), st)
    with pytest.raises(ValueError, match="state must have shape"):
        gdn.decode_commit(snaps, acc, torch.zeros(N, HV, DV, 64))
    with pytest.raises(ValueError, match="bad_count"):
        gdn.decode_commit(snaps, acc, st, bad_count=torch.zeros(0, dtype=torch.int32))


def test_stream_of_another_device_is_rejected():
    """The library launches on the stream it is given with pointers into the
    tensors' device: a stream of another device is refused in the binding,
    and without one the tensors' own device's current stream is used."""
    import types
    from linear_attention_sequence_sm_b200 import gdn
    other = types.SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=77)
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        gdn._stream_handle(other, torch.device("cuda", 0))
    same = types.SimpleNamespace(device=torch.device("cuda", 0), cuda_stream=1234)
    assert gdn._stream_handle(same, torch.device("cuda", 0)).value == 1234
