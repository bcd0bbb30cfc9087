"""GPU: the staged prefill equals the fused call, and a bounded device wait that runs
out is reported through the status word while the context stays usable."""
import numpy as np
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import run_prefill, to_device

pytestmark = pytest.mark.gpu


def test_staged_prefill_equals_kda_prefill_bitwise():
    inp = synthetic.make_prefill_inputs([300, 64, 1, 129], 3, 128, 128, torch.bfloat16, 3.0, 0.02, 77)
    out_ref, fin_ref = run_prefill(inp)
    d = to_device(inp)
    T, H, D = d["q"].shape
    N = d["cu_seqlens"].shape[0] - 1
    ws = torch.empty(kda.kda_prefill_workspace_size(T, N, H, D, D, 64, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(N, H, D, D, device="cuda")
    kda.kda_prefill_prepare(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], ws)
    kda.kda_prefill_scan(out, d["cu_seqlens"], ws, initial_state=d["s0"], final_state=fin)
    assert kda.kda_get_device_status() == kda.KDA_OK
    np.testing.assert_array_equal(out.double().cpu().numpy(), out_ref)
    np.testing.assert_array_equal(fin.double().cpu().numpy(), fin_ref)


def test_expired_bounded_wait_is_reported_and_context_survives():
    assert kda.kda_get_device_status() == kda.KDA_OK
    kda.kda_selftest_bounded_wait(20_000_000)          # 20 ms on a barrier nobody signals
    assert kda.kda_get_device_status() == kda.KDA_ERR_TIMEOUT
    assert kda.kda_get_device_status() == kda.KDA_OK    # cleared by the read
    # the context is still usable: a normal prefill runs and matches its own rerun
    inp = synthetic.make_prefill_inputs([100], 2, 128, 128, torch.bfloat16, 3.0, 0.0, 5)
    o1, f1 = run_prefill(inp)
    o2, f2 = run_prefill(inp)
    np.testing.assert_array_equal(o1, o2)
