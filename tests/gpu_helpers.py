"""Helpers for the GPU parity tests: run libkda on seeded inputs, run the oracle on the
same bytes, compare with the tolerance the method states (max relative Frobenius error
per (sequence, head): 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with fp32 state)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from linear_attention_rule_b200 import kda

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to_device(d: dict) -> dict:
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def run_prefill(inp: dict, C: int = 64, initial=True, want_final=True, workspace=None, in_flags=0):
    """Run kda_prefill (kda_prefill_ex when in_flags is given) on CPU-drawn inputs; returns
    (out fp64 numpy, final fp64 numpy|None)."""
    d = to_device(inp)
    T, H, _ = d["q"].shape
    dv = d["v"].shape[2]
    N = d["cu_seqlens"].shape[0] - 1
    dk = d["q"].shape[2]
    out = torch.full((T, H, dv), float("nan"), dtype=d["q"].dtype, device="cuda")
    sf = torch.full((N, H, dk, dv), float("nan"), device="cuda") if want_final else None
    s0 = d["s0"] if initial else None
    if in_flags:
        kda.kda_prefill_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, in_flags,
                           initial_state=s0, final_state=sf, C=C, workspace=workspace)
    else:
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                        initial_state=s0, final_state=sf, C=C, workspace=workspace)
    status = kda.kda_get_device_status()
    assert status == kda.KDA_OK, kda.kda_status_string(status)
    o = out.double().cpu().numpy()
    f = None if sf is None else sf.double().cpu().numpy()
    return o, f


def oracle_prefill(inp: dict, heads=None, initial=True):
    s0 = inp["s0"] if initial else None
    if s0 is not None and heads is not None:
        s0 = s0[:, list(heads)]
    return oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                          s0=s0, heads=heads)


def check_prefill(inp: dict, out, final, heads=None, tol=None, initial=True, chunk=None):
    """Compare GPU results (all heads) with the oracle on `heads` (default all).
    With `chunk` (the chunk size C), every chunk of C rows of every (sequence, head) slice
    is also held to the tolerance on its own, so that a few wrong rows cannot hide in a
    long slice.  Returns (max output error, max final-state error)."""
    tol = TOL[inp["q"].dtype] if tol is None else tol
    o_ref, f_ref = oracle_prefill(inp, heads, initial=initial)
    hs = list(range(inp["q"].shape[1])) if heads is None else list(heads)
    e_out = oracle.max_rel_frobenius_per_slice(out[:, hs], o_ref, inp["cu_seqlens"])
    e_fin = oracle.max_rel_frobenius_states(final[:, hs], f_ref) if final is not None else 0.0
    assert np.isfinite(out[:, hs]).all()
    assert e_out <= tol, ("output", e_out, tol)
    assert e_fin <= tol, ("final state", e_fin, tol)
    if chunk is not None:
        e_chunk = oracle.max_rel_frobenius_per_chunk(out[:, hs], o_ref, inp["cu_seqlens"], chunk)
        print("worst chunk rel err %.3g" % e_chunk)
        assert e_chunk <= tol, ("output chunk", e_chunk, tol)
    return e_out, e_fin
