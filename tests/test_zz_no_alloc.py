"""kda_prefill_noalloc: the prefill entry point that allocates nothing.

Some callers of this library cannot give kda_prefill a workspace: their device memory
belongs to another allocator (a serving engine that reserved nearly all HBM for its own
pools), or they run where a cudaMalloc stall or cudaFree's device-wide synchronisation
is not acceptable.  kda_prefill_noalloc serves them from a scratch array held inside the
library.  These tests call it through the C-ABI and compare it with kda_prefill (caller
workspace) on two calls in a row, so the second call also shows that what the first
call left in the shared scratch does not leak into its result.

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, run_prefill, to_device

pytestmark = pytest.mark.gpu


def _noalloc(inp):
    d = to_device(inp)
    T, H, dk = d["q"].shape
    N = d["cu_seqlens"].shape[0] - 1
    out = torch.full((T, H, dk), float("nan"), dtype=d["q"].dtype, device="cuda")
    fin = torch.full((N, H, dk, dk), float("nan"), device="cuda")
    kda.kda_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                            initial_state=d["s0"], final_state=fin, C=64)
    assert kda.kda_get_device_status() == kda.KDA_OK
    return out.double().cpu().numpy(), fin.double().cpu().numpy()


def test_noalloc_matches_workspace_prefill_on_two_calls():
    tol = TOL[torch.bfloat16]
    cases = [([700, 333, 64], 4, 401), ([129, 1, 900], 6, 402)]
    for lens, H, seed in cases:
        inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, 3.0, 0.02, seed)
        ref_out, ref_fin = run_prefill(inp)          # kda_prefill with a torch workspace
        out, fin = _noalloc(inp)
        assert oracle.max_rel_frobenius_per_slice(out, ref_out, inp["cu_seqlens"]) <= tol
        assert oracle.max_rel_frobenius_states(fin, ref_fin) <= tol


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = kda.load()
    P = ctypes.c_void_p
    args = lambda T, H, dt, dk: (P(4096), P(4096), P(4096), P(4096), P(4096), None, P(4096), 1,
                                 T, H, dk, dk, dt, P(4096), None, 64, None)
    need = lambda T, H: kda.kda_prefill_workspace_size(T, 1, H, 128, 128, 64, torch.bfloat16)
    assert need(1471, 32) <= kda.NOALLOC_SCRATCH_BYTES < need(1472, 32)
    assert lib.kda_prefill_noalloc(*args(1472, 32, kda.KDA_BF16, 128)) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_prefill_noalloc(*args(1 << 20, 32, kda.KDA_BF16, 128)) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_prefill_noalloc(*args(256, 2, kda.KDA_F32, 64)) == kda.KDA_ERR_UNSUPPORTED
