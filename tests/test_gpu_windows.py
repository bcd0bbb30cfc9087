"""The prefill in windows of chunks: with a workspace below kda_prefill_workspace_size
the chunks are prepared and run a window at a time, and a sequence that crosses a window
boundary carries its fp32 state to the next window.  Nothing of the arithmetic changes,
so every result must equal the one-window run bit for bit: outputs, final states,
emitted states, and the strongly decayed chunks that the CUDA-core preparation handles.
Sequence lengths put empty sequences at the start, in the middle and at the very end, and
boundaries inside sequences, at their first and at their last chunk."""
import numpy as np
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import check_prefill, run_prefill, to_device

pytestmark = pytest.mark.gpu

REC = 90624   # bytes of one chunk record (64 tokens of one head)


def _workspace(lens, H, window):
    """A workspace that holds records for `window` chunks (plus the fixed part)."""
    T, N = sum(lens), len(lens)
    least = kda.kda_prefill_workspace_size_min(T, N, H, 128, 128, 64, torch.bfloat16)
    ws = least + (window - 8) * H * (REC + 8) + 2048   # (the layout's alignment slack)
    n = kda.kda_prefill_windows(T, N, H, 128, 128, 64, torch.bfloat16, ws)
    assert n > 1, (lens, H, window, n)
    return torch.empty(ws, dtype=torch.uint8, device="cuda"), n


@pytest.mark.parametrize("window", [8, 13, 40])
def test_windows_equal_one_window_varlen(window):
    lens = [0, 700, 64, 0, 1, 2000, 129, 63, 0]
    H = 3
    inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, 3.0, 0.02, 700 + window)
    ws, n = _workspace(lens, H, window)
    ref_out, ref_fin = run_prefill(inp, in_flags=kda.KDA_IN_SERIAL_CHAINS)
    out, fin = run_prefill(inp, workspace=ws)
    np.testing.assert_array_equal(out, ref_out)
    np.testing.assert_array_equal(fin, ref_fin)
    if window == 13:   # and against the oracle, per slice and per chunk
        check_prefill(inp, out, fin, chunk=64)


def test_windows_one_long_sequence_without_initial_state():
    lens = [64 * 100 + 17]
    H = 4
    inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, 3.0, 0.0, 711)
    ws, n = _workspace(lens, H, 9)
    assert n == 12
    for initial in (False, True):
        ref_out, ref_fin = run_prefill(inp, initial=initial, in_flags=kda.KDA_IN_SERIAL_CHAINS)
        out, fin = run_prefill(inp, initial=initial, workspace=ws)
        np.testing.assert_array_equal(out, ref_out)
        np.testing.assert_array_equal(fin, ref_fin)
    # no final state requested: the state still crosses the windows through the workspace
    out, _ = run_prefill(inp, want_final=False, workspace=ws)
    np.testing.assert_array_equal(out, ref_out)


def test_windows_strong_decay_and_emission():
    """Strongly decayed chunks (g = logsigmoid(N(-3, 1))) are listed per window; emitted
    states at chunk boundaries are written from whichever window holds them."""
    lens = [900, 0, 1300, 64]
    H = 2
    inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, -3.0, 0.02, 712)
    d = to_device(inp)
    T, N = sum(lens), len(lens)
    ws, n = _workspace(lens, H, 10)
    pos = torch.tensor([64, 896, 900, 900 + 640, 2200, 2264], dtype=torch.int64, device="cuda")
    res = []
    for workspace, flags in ((None, kda.KDA_IN_SERIAL_CHAINS), (ws, 0)):
        out = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        fin = torch.full((N, H, 128, 128), float("nan"), device="cuda")
        em = torch.full((pos.shape[0], H, 128, 128), float("nan"), device="cuda")
        kda.kda_prefill_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, flags,
                           initial_state=d["s0"], final_state=fin, emit_pos=pos, emit_states=em,
                           workspace=workspace)
        assert kda.kda_get_device_status() == kda.KDA_OK
        res.append([x.double().cpu().numpy() for x in (out, fin, em)])
    for a, b in zip(*res):
        np.testing.assert_array_equal(b, a)
    check_prefill(inp, res[1][0], res[1][1])


def test_windows_below_the_least_workspace_is_rejected():
    lens = [4096]
    least = kda.kda_prefill_workspace_size_min(4096, 1, 2, 128, 128, 64, torch.bfloat16)
    inp = synthetic.make_prefill_inputs(lens, 2, 128, 128, torch.bfloat16, 3.0, 0.0, 713)
    ws = torch.empty(least - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KdaError):
        run_prefill(inp, workspace=ws)
