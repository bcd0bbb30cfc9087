"""CPU checks of the Python binding's tensor validation: a wrong dtype, shape, layout or
device raises in Python before any pointer reaches the library (a CPU tensor handed to
a kernel, or a tensor smaller than the sizes say, would be an out-of-bounds access on the
GPU).  No GPU is needed: every case fails before the library call."""
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_rule_b200 import build
    build.build()
    kda.load()


def _prefill_args(dtype=torch.bfloat16, D=128, H=2, lens=(70, 5)):
    inp = synthetic.make_prefill_inputs(list(lens), H, D, D, dtype, 3.0, 0.02, 3)
    T, N = sum(lens), len(lens)
    out = torch.empty(T, H, D, dtype=dtype)
    fin = torch.empty(N, H, D, D)
    return inp, out, fin


def _call_prefill(inp, out_, fin_, **over):
    a = dict(inp, out=out_, fin=fin_)
    a.update(over)
    kda.kda_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu_seqlens"], a["out"],
                    initial_state=a["s0"], final_state=a["fin"])


def test_valid_shapes_on_the_cpu_fail_only_for_the_device():
    inp, out, fin = _prefill_args()
    with pytest.raises(ValueError, match="must be on"):
        _call_prefill(inp, out, fin)


@pytest.mark.parametrize("key,bad,exc", [
    ("g", lambda t: t.to(torch.bfloat16), TypeError),          # the gate is fp32
    ("beta", lambda t: t.double(), TypeError),
    ("cu_seqlens", lambda t: t.long(), TypeError),            # int32 offsets
    ("out", lambda t: t.float(), TypeError),                  # out in q's dtype
    ("k", lambda t: t[:-1].contiguous(), ValueError),         # one token short
    ("g", lambda t: t[:, :, :64].contiguous(), ValueError),   # fewer channels than q
    ("beta", lambda t: t[:, :1].contiguous(), ValueError),    # fewer heads
    ("s0", lambda t: t[:1].contiguous(), ValueError),         # states of one sequence only
    ("fin", lambda t: t.transpose(2, 3), ValueError),         # not contiguous
])
def test_prefill_rejects_mismatched_tensors(key, bad, exc):
    inp, out, fin = _prefill_args()
    cur = {"out": out, "fin": fin}.get(key, inp.get(key))
    with pytest.raises(exc):
        _call_prefill(inp, out, fin, **{key: bad(cur)})


def test_scalar_gate_entry_points_take_one_gate_per_token_and_head():
    inp, out, fin = _prefill_args()
    with pytest.raises(ValueError, match="shape"):   # a per-channel gate given to the GDN entry
        kda.kda_prefill_gdn(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                            out, initial_state=inp["s0"], final_state=fin)
    g1 = inp["g"][:, :, 0].contiguous()
    with pytest.raises(ValueError, match="must be on"):
        kda.kda_prefill_ex(inp["q"], inp["k"], inp["v"], g1, inp["beta"], inp["cu_seqlens"], out,
                           kda.KDA_IN_G_SCALAR, initial_state=inp["s0"], final_state=fin)
    with pytest.raises(ValueError, match="shape"):   # without the flag g must be per channel
        kda.kda_prefill_ex(inp["q"], inp["k"], inp["v"], g1, inp["beta"], inp["cu_seqlens"], out,
                           0, initial_state=inp["s0"], final_state=fin)


def test_emission_tensors_are_checked():
    inp, out, fin = _prefill_args()
    pos = torch.tensor([64], dtype=torch.int64)
    with pytest.raises(ValueError, match="shape"):   # one position, two state slots
        kda.kda_prefill_emit(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                             out, pos, torch.empty(2, 2, 128, 128), initial_state=inp["s0"])
    with pytest.raises(TypeError):
        kda.kda_prefill_emit(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                             out, pos.int(), torch.empty(1, 2, 128, 128), initial_state=inp["s0"])
    with pytest.raises(ValueError, match="together"):
        kda.kda_prefill_ex(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                           out, 0, emit_pos=pos)


def test_decode_rejects_mismatched_tensors():
    N, H, D = 3, 2, 64
    x = synthetic.make_decode_step_inputs(N, H, D, D, torch.float32, 3.0, 5, 0)
    S = synthetic.make_decode_state(N, H, D, D, 0.02, 5)
    out = torch.empty(N, H, D)
    with pytest.raises(ValueError, match="must be on"):
        kda.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out)
    with pytest.raises(ValueError, match="shape"):
        kda.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], S[:, :, :32].contiguous(), out)
    with pytest.raises(TypeError):
        kda.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], S.double(), out)
    with pytest.raises(ValueError, match="shape"):
        kda.kda_decode_gdn(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out)
    with pytest.raises(TypeError):
        kda.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], S, out.to(torch.bfloat16))
