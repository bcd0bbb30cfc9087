"""GPU: the fused input prologue (kda_prefill_ex / kda_decode_ex with KDA_IN_* flags) on raw
layer inputs, against the fp64 oracle given the inputs transformed by the oracle's own
fp64 prologue (oracle.prologue: q / max(||q||, 1e-12), the same for k, logsigmoid of the
gate logits, sigmoid of the beta logits) from the same bytes."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, to_device

pytestmark = pytest.mark.gpu

ALL = kda.KDA_IN_NORMALIZE_QK | kda.KDA_IN_G_LOGITS | kda.KDA_IN_BETA_LOGITS


def _transformed(raw, flags, scalar_gate=False):
    """oracle.prologue on the raw inputs; fp64 arrays for the oracle's recurrence (which
    reads its inputs as fp32, so they are handed over rounded to fp32)."""
    q, k, g, b = oracle.prologue(raw["q"], raw["k"], raw["g"], raw["beta"],
                                 bool(flags & kda.KDA_IN_NORMALIZE_QK),
                                 bool(flags & kda.KDA_IN_G_LOGITS),
                                 bool(flags & kda.KDA_IN_BETA_LOGITS))
    if scalar_gate:
        g = np.broadcast_to(g[..., None], g.shape + (q.shape[-1],))
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return {"q": f32(q), "k": f32(k), "v": raw["v"].float(), "g": f32(g), "beta": f32(b)}


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 64)])
@pytest.mark.parametrize("flags", [ALL, kda.KDA_IN_NORMALIZE_QK, kda.KDA_IN_G_LOGITS | kda.KDA_IN_BETA_LOGITS])
def test_prefill_prologue_matches_oracle(dtype, D, flags):
    lens = [200, 64, 1, 0, 70]
    raw = synthetic.make_raw_prefill_inputs(lens, 3, D, D, dtype, 3.0, 0.02, 121 + D + flags)
    if not flags & kda.KDA_IN_NORMALIZE_QK:  # then q and k must arrive normalised (the method
        for key in ("q", "k"):                # assumes unit keys: the delta rule is unstable without)
            raw[key] = torch.from_numpy(oracle.l2_normalize(raw[key])).to(dtype)
    if not flags & kda.KDA_IN_G_LOGITS:      # then g must already be a log-decay
        raw["g"] = torch.from_numpy(oracle.logsigmoid(raw["g"])).float()
    if not flags & kda.KDA_IN_BETA_LOGITS:
        raw["beta"] = torch.from_numpy(oracle.sigmoid(raw["beta"])).float()
    d = to_device(raw)
    T = d["q"].shape[0]
    out = torch.full((T, 3, D), float("nan"), dtype=dtype, device="cuda")
    fin = torch.full((len(lens), 3, D, D), float("nan"), device="cuda")
    kda.kda_prefill_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, flags,
                       initial_state=d["s0"], final_state=fin)
    assert kda.kda_get_device_status() == kda.KDA_OK
    t = _transformed(raw, flags)
    o_ref, f_ref = oracle.prefill(t["q"], t["k"], t["v"], t["g"], t["beta"], raw["cu_seqlens"], s0=raw["s0"])
    tol = TOL[dtype]
    assert oracle.max_rel_frobenius_per_slice(out.double().cpu().numpy(), o_ref, raw["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin.double().cpu().numpy(), f_ref) <= tol


def test_prefill_prologue_with_scalar_gate_and_emission():
    lens = [300, 65]
    raw = synthetic.make_raw_prefill_inputs(lens, 2, 128, 128, torch.bfloat16, 3.0, 0.02, 131,
                                            scalar_gate=True)
    d = to_device(raw)
    out = torch.empty(365, 2, 128, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(2, 2, 128, 128, device="cuda")
    pos = torch.tensor([128, 365], dtype=torch.int64, device="cuda")   # 365: end of sequence 1
    es = torch.full((2, 2, 128, 128), float("nan"), device="cuda")
    kda.kda_prefill_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                       ALL | kda.KDA_IN_G_SCALAR, initial_state=d["s0"], final_state=fin,
                       emit_pos=pos, emit_states=es)
    assert kda.kda_get_device_status() == kda.KDA_OK
    t = _transformed(raw, ALL, scalar_gate=True)
    o_ref, f_ref = oracle.prefill(t["q"], t["k"], t["v"], t["g"], t["beta"], raw["cu_seqlens"], s0=raw["s0"])
    tol = TOL[torch.bfloat16]
    assert oracle.max_rel_frobenius_per_slice(out.double().cpu().numpy(), o_ref, raw["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin.double().cpu().numpy(), f_ref) <= tol
    sl = slice(0, 128)   # emission 0: sequence 0 after its first 128 tokens
    _, f128 = oracle.prefill(t["q"][sl], t["k"][sl], t["v"][sl], t["g"][sl], t["beta"][sl],
                             torch.tensor([0, 128], dtype=torch.int32), s0=raw["s0"][0:1])
    assert oracle.max_rel_frobenius_states(es[0:1].double().cpu().numpy(), f128) <= tol
    np.testing.assert_array_equal(es[1].double().cpu().numpy(), fin[1].double().cpu().numpy())


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("scalar_gate", [False, True])
def test_decode_prologue_matches_oracle(dtype, D, scalar_gate):
    N, H, steps = 5, 3, 4
    S = synthetic.make_decode_state(N, H, D, D, 0.02, 141).cuda()
    S_ref = S.double().cpu().numpy()
    flags = ALL | (kda.KDA_IN_G_SCALAR if scalar_gate else 0)
    for step in range(steps):
        raw = synthetic.make_raw_prefill_inputs([1] * N, H, D, D, dtype, 3.0, 0.0, 141 + 7 * step,
                                                scalar_gate=scalar_gate)
        d = {k: v.cuda() for k, v in raw.items() if k in ("q", "k", "v", "g", "beta")}
        out = torch.empty(N, H, D, dtype=dtype, device="cuda")
        kda.kda_decode_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], S, out, flags)
        t = _transformed(raw, ALL, scalar_gate=scalar_gate)
        o_ref, S_ref = oracle.decode(t["q"], t["k"], t["v"], t["g"], t["beta"], S_ref)
        assert oracle.rel_frobenius(out.double().cpu().numpy(), o_ref) <= TOL[dtype]
    assert kda.kda_get_device_status() == kda.KDA_OK
    assert oracle.max_rel_frobenius_states(S.double().cpu().numpy(), S_ref) <= TOL[dtype]
