"""GPU: state emission for a prefix cache (kda_prefill_emit), through the C-ABI.  Every
emitted state is compared with the fp64 oracle run on the truncated sequence (the plain
definition of "the state after this prefix"); the outputs and final states must equal
kda_prefill's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, run_prefill, to_device

pytestmark = pytest.mark.gpu

LENS = [300, 64, 129, 1]     # cu_seqlens 0, 300, 364, 493, 494
H = 4


def _emit(inp, pos):
    d = to_device(inp)
    T = d["q"].shape[0]
    N = len(LENS)
    out = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    fin = torch.full((N, H, 128, 128), float("nan"), device="cuda")
    emit_pos = torch.tensor(pos, dtype=torch.int64, device="cuda")
    es = torch.full((len(pos), H, 128, 128), float("nan"), device="cuda")
    kda.kda_prefill_emit(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                         emit_pos, es, initial_state=d["s0"], final_state=fin)
    status = kda.kda_get_device_status()
    return status, out.double().cpu().numpy(), fin.double().cpu().numpy(), es.double().cpu().numpy()


def _prefix_state(inp, n, t):
    """fp64 oracle state of sequence n after its tokens cu[n] .. t-1."""
    cu = inp["cu_seqlens"].tolist()
    a = cu[n]
    sl = slice(a, t)
    _, f = oracle.prefill(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["g"][sl], inp["beta"][sl],
                          torch.tensor([0, t - a], dtype=torch.int32), s0=inp["s0"][n:n + 1])
    return f[0]


def test_emitted_states_are_the_prefix_states():
    inp = synthetic.make_prefill_inputs(LENS, H, 128, 128, torch.bfloat16, 3.0, 0.02, 71)
    # chunk ends inside sequences, a partial last chunk's end, full-chunk sequence ends
    pos = [64, 192, 300, 364, 364 + 128, 493, 494]
    seq_of = [0, 0, 0, 1, 2, 2, 3]
    status, out, fin, es = _emit(inp, pos)
    assert status == kda.KDA_OK, kda.kda_status_string(status)
    o_ref, f_ref = run_prefill(inp)
    np.testing.assert_array_equal(out, o_ref)
    np.testing.assert_array_equal(fin, f_ref)
    for e, (t, n) in enumerate(zip(pos, seq_of)):
        ref = _prefix_state(inp, n, t)
        err = oracle.max_rel_frobenius_states(es[e:e + 1], ref[None])
        assert err <= TOL[torch.bfloat16], (t, err)
    # an emission at a sequence's end is that sequence's final state, bit for bit
    for e, n in ((2, 0), (3, 1), (5, 2), (6, 3)):
        np.testing.assert_array_equal(es[e], fin[n])


def test_bad_emission_position_is_reported_and_others_still_written():
    inp = synthetic.make_prefill_inputs(LENS, H, 128, 128, torch.bfloat16, 3.0, 0.02, 72)
    pos = [128, 65, 0, 495, 300]   # 65: inside a chunk; 0: no token before it; 495: past the end
    status, _, fin, es = _emit(inp, pos)
    assert status == kda.KDA_ERR_BAD_EMIT_POS
    assert kda.kda_get_device_status() == kda.KDA_OK    # cleared by the read
    assert np.isnan(es[1]).all() and np.isnan(es[2]).all() and np.isnan(es[3]).all()
    np.testing.assert_array_equal(es[4], fin[0])
    err = oracle.max_rel_frobenius_states(es[0:1], _prefix_state(inp, 0, 128)[None])
    assert err <= TOL[torch.bfloat16]


def test_no_emission_positions_is_plain_prefill():
    inp = synthetic.make_prefill_inputs(LENS, H, 128, 128, torch.bfloat16, 3.0, 0.02, 73)
    status, out, fin, es = _emit(inp, [])
    assert status == kda.KDA_OK
    o_ref, f_ref = run_prefill(inp)
    np.testing.assert_array_equal(out, o_ref)
    np.testing.assert_array_equal(fin, f_ref)
