"""The prefill captured in a CUDA graph: its kernels depend on one another through the
stream (programmatic dependent launch between the chunk table, the preparations and the
recurrence), and a small workspace adds the loop over windows.  A captured call, replayed
on new input contents, must give the bits an eager call gives on those contents: with the
full workspace, with a workspace of a few windows, and through the allocation-free entry
point (whose first call in a context comes before any capture)."""
import numpy as np
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic

pytestmark = pytest.mark.gpu

LENS, H = [700, 333, 0, 1000], 4


def _inputs(seed):
    inp = synthetic.make_prefill_inputs(LENS, H, 128, 128, torch.bfloat16, 3.0, 0.02, seed)
    return {k: (None if v is None else v.cuda()) for k, v in inp.items()}


def _buffers(d):
    T, N = sum(LENS), len(LENS)
    out = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    fin = torch.full((N, H, 128, 128), float("nan"), device="cuda")
    return out, fin


def _call(kind, d, out, fin, ws):
    if kind == "noalloc":
        kda.kda_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                                initial_state=d["s0"], final_state=fin)
    else:
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                        initial_state=d["s0"], final_state=fin, workspace=ws)


def _workspace(kind):
    T, N = sum(LENS), len(LENS)
    if kind == "noalloc":
        return None
    full = kda.kda_prefill_workspace_size(T, N, H, 128, 128, 64, torch.bfloat16)
    least = kda.kda_prefill_workspace_size_min(T, N, H, 128, 128, 64, torch.bfloat16)
    size = full if kind == "full" else least + 4 * H * (90624 + 8) + 2048
    n = kda.kda_prefill_windows(T, N, H, 128, 128, 64, torch.bfloat16, size)
    assert (n == 1) == (kind == "full"), n
    return torch.empty(size, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("kind", ["full", "windows", "noalloc"])
def test_prefill_replayed_from_a_graph_matches_eager(kind):
    ws = _workspace(kind)
    d = _inputs(900)
    out, fin = _buffers(d)
    _call(kind, d, out, fin, ws)   # eager first (also the first allocation-free call here)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == kda.KDA_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _call(kind, d, out, fin, ws)
    for seed in (901, 902):
        new = _inputs(seed)
        for key in ("q", "k", "v", "g", "beta", "s0"):
            d[key].copy_(new[key])
        out.fill_(float("nan"))
        fin.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == kda.KDA_OK
        got = out.double().cpu().numpy(), fin.double().cpu().numpy()
        ref_out, ref_fin = _buffers(new)
        _call(kind, new, ref_out, ref_fin, ws)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == kda.KDA_OK
        np.testing.assert_array_equal(got[0], ref_out.double().cpu().numpy())
        np.testing.assert_array_equal(got[1], ref_fin.double().cpu().numpy())
        assert not np.isnan(got[0]).any()
