"""GPU: the chunk-parallel scan of the recurrence (few long chains: each (sequence, head)
chain cut into segments whose affine transitions are composed), against the fp64 oracle
and against the serial chains on the same inputs (KDA_IN_SERIAL_CHAINS).

The scan is chosen by the library from the sizes alone (kda_prefill_workspace_size): it
runs where sequences x heads leave most SMs idle and segments stay long enough."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, check_prefill, run_prefill, to_device

pytestmark = pytest.mark.gpu


def _serial_vs_scan(inp):
    out_scan, fin_scan = run_prefill(inp)
    out_ser, fin_ser = run_prefill(inp, in_flags=kda.KDA_IN_SERIAL_CHAINS)
    tol = TOL[torch.bfloat16]
    assert oracle.max_rel_frobenius_per_slice(out_scan, out_ser, inp["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin_scan, fin_ser) <= tol
    return out_scan, fin_scan


@pytest.mark.parametrize("H", [4, 8])
def test_scan_few_heads_long_sequence(H):
    """T = 2^18 tokens, H = 4 or 8 heads: 4096 chunks per chain, cut into segments; every
    output row and the final state of every head against the oracle."""
    T = 1 << 18
    assert kda.kda_prefill_launches(T, 1, H, 128, 128, 64, torch.bfloat16) == 7   # the scan runs
    inp = synthetic.make_prefill_inputs([T], H, 128, 128, torch.bfloat16, 3.0, 0.02, 500 + H)
    out, fin = _serial_vs_scan(inp)
    e_o, e_f = check_prefill(inp, out, fin, chunk=64)
    print("scan H=%d T=%d max rel err out %.3g final %.3g" % (H, T, e_o, e_f))


def test_scan_d64():
    """The scan at d = 64 (the tensor-core kernels on the first 64 channels of a
    128-channel problem): T = 2^17, H = 4, with an initial state, against the oracle and
    against the serial chains."""
    T, H = 1 << 17, 4
    assert kda.kda_prefill_launches(T, 1, H, 64, 64, 64, torch.bfloat16) == 7   # the scan runs
    inp = synthetic.make_prefill_inputs([T], H, 64, 64, torch.bfloat16, 3.0, 0.02, 520)
    out, fin = _serial_vs_scan(inp)
    e_o, e_f = check_prefill(inp, out, fin, chunk=64)
    print("scan d=64 H=%d T=%d max rel err out %.3g final %.3g" % (H, T, e_o, e_f))


def test_scan_varlen_mixed_lengths_and_emission():
    """Sequences of 420000, 200000, 0 and 1 tokens at H = 1: the long ones are cut into
    segments, the empty and the one-token sequence are one segment each.  States emitted
    inside and at the end of the long sequence, and in the second one, match the oracle."""
    lens = [420000, 200000, 0, 1]
    H = 1
    T = sum(lens)
    assert kda.kda_prefill_launches(T, 4, H, 128, 128, 64, torch.bfloat16) == 8   # the scan runs (+1: the order of the 4 sequences)
    inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, 3.0, 0.02, 510)
    out, fin = _serial_vs_scan(inp)
    check_prefill(inp, out, fin, chunk=64)
    d = to_device(inp)
    pos = torch.tensor([64 * 2500, 420000, 420000 + 64 * 7], dtype=torch.int64, device="cuda")
    es = torch.full((3, H, 128, 128), float("nan"), device="cuda")
    out2 = torch.empty_like(d["v"])
    kda.kda_prefill_emit(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out2, pos, es,
                         initial_state=d["s0"])
    assert kda.kda_get_device_status() == kda.KDA_OK
    es = es.double().cpu().numpy()
    tol = TOL[torch.bfloat16]
    for e, (seq, t_end) in enumerate([(0, 64 * 2500), (0, 420000), (1, 64 * 7)]):
        a = sum(lens[:seq])
        sl = slice(a, a + t_end)
        _, f_ref = oracle.prefill(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["g"][sl], inp["beta"][sl],
                                  torch.tensor([0, t_end], dtype=torch.int32), s0=inp["s0"][seq:seq + 1])
        assert oracle.max_rel_frobenius_states(es[e:e + 1], f_ref) <= tol, e
