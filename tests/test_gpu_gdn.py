"""GPU: the Gated DeltaNet entry points (one log-decay per token and head), through the C-ABI.
A scalar gate is the diagonal gate with every entry equal, so the oracle runs the KDA
recurrence on the gate broadcast over the key channels; the tensor-core path must also equal
kda_prefill given that broadcast gate, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, to_device

pytestmark = pytest.mark.gpu


def _gdn_inputs(lens, H, D, dtype, seed):
    inp = synthetic.make_prefill_inputs(lens, H, D, D, dtype, 3.0, 0.02, seed)
    inp["g1"] = inp["g"][:, :, 0].contiguous()                      # scalar gate [T, H]
    inp["g"] = inp["g1"][:, :, None].expand_as(inp["g"]).contiguous()  # the same, per channel
    return inp


def _run(fn, inp, g):
    d = to_device(inp)
    T, H, D = d["q"].shape
    N = d["cu_seqlens"].shape[0] - 1
    out = torch.full((T, H, D), float("nan"), dtype=d["q"].dtype, device="cuda")
    fin = torch.full((N, H, D, D), float("nan"), device="cuda")
    fn(d["q"], d["k"], d["v"], g.cuda(), d["beta"], d["cu_seqlens"], out, initial_state=d["s0"],
       final_state=fin)
    assert kda.kda_get_device_status() == kda.KDA_OK
    return out.double().cpu().numpy(), fin.double().cpu().numpy()


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 64)])
def test_gdn_prefill_matches_oracle(dtype, D):
    lens = [300, 64, 1, 0, 129]
    inp = _gdn_inputs(lens, 4, D, dtype, 81 + D)
    out, fin = _run(kda.kda_prefill_gdn, inp, inp["g1"])
    o_ref, f_ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  inp["cu_seqlens"], s0=inp["s0"])
    tol = TOL[dtype]
    assert oracle.max_rel_frobenius_per_slice(out, o_ref, inp["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin, f_ref) <= tol


def test_gdn_prefill_equals_kda_with_broadcast_gate_bitwise():
    inp = _gdn_inputs([500, 77], 3, 128, torch.bfloat16, 91)
    o_gdn, f_gdn = _run(kda.kda_prefill_gdn, inp, inp["g1"])
    o_kda, f_kda = _run(kda.kda_prefill, inp, inp["g"])
    np.testing.assert_array_equal(o_gdn, o_kda)
    np.testing.assert_array_equal(f_gdn, f_kda)


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_gdn_decode_matches_oracle(dtype, D):
    N, H, steps = 6, 4, 5
    S = synthetic.make_decode_state(N, H, D, D, 0.02, 95).cuda()
    S_ref = S.double().cpu().numpy()
    for step in range(steps):
        x = synthetic.make_decode_step_inputs(N, H, D, D, dtype, 3.0, 95, step)
        g1 = x["g"][:, :, 0].contiguous()
        gb = g1[:, :, None].expand_as(x["g"]).contiguous()
        d = {k: v.cuda() for k, v in x.items()}
        out = torch.empty(N, H, D, dtype=dtype, device="cuda")
        kda.kda_decode_gdn(d["q"], d["k"], d["v"], g1.cuda(), d["beta"], S, out)
        o_ref, S_ref = oracle.decode(x["q"], x["k"], x["v"], gb, x["beta"], S_ref)
        assert oracle.rel_frobenius(out.double().cpu().numpy(), o_ref) <= TOL[dtype]
    assert kda.kda_get_device_status() == kda.KDA_OK
    assert oracle.max_rel_frobenius_states(S.double().cpu().numpy(), S_ref) <= TOL[dtype]
