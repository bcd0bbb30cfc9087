"""kda_prefill_noalloc: the prefill entry point that allocates nothing.

Some callers of this library cannot give kda_prefill a workspace: their device memory
belongs to another allocator (a serving engine that reserved nearly all HBM for its own
pools), or they run where a cudaMalloc stall or cudaFree's device-wide synchronisation
is not acceptable.  kda_prefill_noalloc serves them from a scratch array held inside the
library.  These tests call it through the C-ABI and compare it with kda_prefill (caller
workspace), bit for bit, on calls in a row: the first fills the scratch nearly to its
limit, so the later, smaller calls show that what an earlier call left in the shared
scratch does not leak into their results.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import run_prefill, to_device

pytestmark = pytest.mark.gpu


def _need(T, H, N=1):
    return kda.kda_prefill_workspace_size(T, N, H, 128, 128, 64, torch.bfloat16)


def _largest_tokens_that_fit(H):
    """Largest one-sequence length whose full workspace (one window) fits the static
    scratch (bisection on the library's own workspace size)."""
    lo, hi = 0, 1
    while _need(hi, H) <= kda.NOALLOC_SCRATCH_BYTES:
        lo, hi = hi, 2 * hi
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if _need(mid, H) <= kda.NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo


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


def test_noalloc_matches_workspace_prefill_on_calls_in_a_row():
    """The same kernels on the same inputs as kda_prefill, only the workspace differs, so
    the results must be identical bit for bit.  The first call is larger than the scratch
    and runs in windows of chunks; the second fills the scratch in one window almost to
    its limit; the smaller calls after them run over what those left there (the chunk
    table, the records, the carried states and beyond), which must not leak into their
    results."""
    T_max = _largest_tokens_that_fit(32)
    assert _need(T_max, 32) > kda.NOALLOC_SCRATCH_BYTES * 0.95
    windows = lambda lens, H: kda.kda_prefill_windows(sum(lens), len(lens), H, 128, 128, 64, torch.bfloat16,
                                                      kda.NOALLOC_SCRATCH_BYTES)
    cases = [([8192], 32, 0.02, 399), ([T_max], 32, 0.0, 400), ([700, 333, 64], 4, 0.02, 401),
             ([129, 1, 900], 6, 0.02, 402)]
    assert windows(*cases[0][:2]) > 4 and windows(*cases[1][:2]) == 1
    for lens, H, s0_std, seed in cases:
        inp = synthetic.make_prefill_inputs(lens, H, 128, 128, torch.bfloat16, 3.0, s0_std, seed)
        ref_out, ref_fin = run_prefill(inp)          # kda_prefill with a full torch workspace
        out, fin = _noalloc(inp)
        np.testing.assert_array_equal(out, ref_out)
        np.testing.assert_array_equal(fin, ref_fin)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Only a problem whose least workspace (windows of 8 chunks) exceeds the scratch is
    refused: with many heads, 8 chunks of records no longer fit."""
    lib = kda.load()
    P = ctypes.c_void_p
    args = lambda T, H, dt, dk: (P(4096), P(4096), P(4096), P(4096), P(4096), None, P(4096), 1,
                                 T, H, dk, dk, dt, P(4096), None, 64, None)
    least = lambda T, H: kda.kda_prefill_workspace_size_min(T, 1, H, 128, 128, 64, torch.bfloat16)
    assert least(1 << 20, 32) <= kda.NOALLOC_SCRATCH_BYTES < least(1 << 20, 128)
    assert lib.kda_prefill_noalloc(*args(1 << 20, 128, kda.KDA_BF16, 128)) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_prefill_noalloc(*args(256, 2, kda.KDA_F32, 64)) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_prefill_noalloc(*args(256, 2, 7, 128)) == kda.KDA_ERR_INVALID_ARG
