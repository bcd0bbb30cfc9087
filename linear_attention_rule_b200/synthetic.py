"""Seeded synthetic inputs for KDA prefill and decode.

This module only draws random inputs; it holds none of the method's arithmetic.
Both the CUDA path (through the tests and the benchmark) and the fp64 oracle
receive the exact tensors it returns, so the two always see identical bytes.

Recipe (the workloads of the five benchmark configurations):
  * q, k, v ~ N(0, 1); q and k are L2-normalised per (token, head) in fp32 and then
    cast to the input dtype (normalisation is part of the layer that feeds KDA,
    "SemiAnalysis Kimi K3", the KDA layer figure: L2 norm on query and key).
  * beta = sigmoid(N(0, 1)), fp32, shape [T, H].
  * g = logsigmoid(N(mu, 1)), fp32, shape [T, H, d_k]  (per-channel log-decay, so the
    decay alpha = exp(g) lies in (0, 1)); mu = 3, or 4 for the slow-decay long context.
  * initial state ~ N(0, s0_std^2) fp32 [N, H, d_k, d_v], or none.

Determinism: every head draws from its own CPU generator, seeded from (seed, head),
in the fixed order q, k, v, beta-logits, g-logits, initial state.  Any subset of
heads can therefore be regenerated alone and equals the corresponding slice of the
full tensors.  Varlen lengths come from a generator seeded with `seed` alone.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

HEAD_SEED_STRIDE = 1_000_003
STEP_SEED_STRIDE = 7_919


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    lengths: Optional[Sequence[int]]   # None -> drawn (varlen)
    H: int
    D: int
    C: int
    dtype: torch.dtype
    g_mean: float
    s0_std: float
    seed: int
    num_seqs: int = 1
    len_range: tuple = (0, 0)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int
    H: int
    D: int
    dtype: torch.dtype
    g_mean: float
    s0_std: float
    steps: int
    seed: int


CONFIGS = {
    0: PrefillConfig("tiny-f32 B=1 H=2 T=256 D=64 C=64", [256], 2, 64, 64,
                     torch.float32, 3.0, 0.0, 1000),
    1: PrefillConfig("prefill B=1 H=32 T=8192 D=128 C=64 bf16", [8192], 32, 128, 64,
                     torch.bfloat16, 3.0, 0.0, 1001),
    2: PrefillConfig("varlen 16 seqs U[1024,32768] H=32 D=128 C=64 bf16 S0~N(0,0.02^2)",
                     None, 32, 128, 64, torch.bfloat16, 3.0, 0.02, 1002,
                     num_seqs=16, len_range=(1024, 32768)),
    3: DecodeConfig("decode N=256 H=32 D=128 bf16 64 steps", 256, 32, 128,
                    torch.bfloat16, 3.0, 0.02, 64, 1003),
    4: PrefillConfig("long prefill B=1 H=32 T=1048576 D=128 C=64 bf16 g~logsigmoid(N(4,1))",
                     [1 << 20], 32, 128, 64, torch.bfloat16, 4.0, 0.0, 1004),
}


def draw_lengths(cfg: PrefillConfig) -> list:
    """Sequence lengths of a prefill config (drawn for the varlen case)."""
    if cfg.lengths is not None:
        return list(cfg.lengths)
    gen = torch.Generator().manual_seed(cfg.seed)
    lo, hi = cfg.len_range
    return [int(x) for x in torch.randint(lo, hi + 1, (cfg.num_seqs,), generator=gen)]


def cu_seqlens_of(lengths: Sequence[int]) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def _l2_normalise(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _head_generator(seed: int, head: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed + HEAD_SEED_STRIDE * (head + 1))


def make_prefill_inputs(lengths: Sequence[int], H: int, dk: int, dv: int,
                        dtype: torch.dtype, g_mean: float, s0_std: float, seed: int,
                        heads: Optional[Sequence[int]] = None,
                        g_scale: float = 1.0) -> dict:
    """Draw one packed varlen prefill batch on the CPU.

    Returns q, k [T, Hs, dk] and v [T, Hs, dv] in `dtype`; g [T, Hs, dk] and
    beta [T, Hs] in fp32; cu_seqlens int32 [N+1]; s0 fp32 [N, Hs, dk, dv] or None,
    where Hs = len(heads) (all H heads when heads is None).
    """
    heads = list(range(H)) if heads is None else list(heads)
    T = int(sum(lengths))
    N = len(lengths)
    Hs = len(heads)
    q = torch.empty(T, Hs, dk, dtype=dtype)
    k = torch.empty(T, Hs, dk, dtype=dtype)
    v = torch.empty(T, Hs, dv, dtype=dtype)
    g = torch.empty(T, Hs, dk, dtype=torch.float32)
    beta = torch.empty(T, Hs, dtype=torch.float32)
    s0 = torch.empty(N, Hs, dk, dv, dtype=torch.float32) if s0_std > 0 else None
    for j, h in enumerate(heads):
        gen = _head_generator(seed, h)
        q[:, j] = _l2_normalise(torch.randn(T, dk, generator=gen)).to(dtype)
        k[:, j] = _l2_normalise(torch.randn(T, dk, generator=gen)).to(dtype)
        v[:, j] = torch.randn(T, dv, generator=gen).to(dtype)
        beta[:, j] = torch.sigmoid(torch.randn(T, generator=gen))
        g[:, j] = torch.nn.functional.logsigmoid(
            g_mean + g_scale * torch.randn(T, dk, generator=gen))
        if s0 is not None:
            s0[:, j] = s0_std * torch.randn(N, dk, dv, generator=gen)
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu_seqlens_of(lengths), s0=s0)


def make_config_inputs(cfg_id: int, heads: Optional[Sequence[int]] = None) -> dict:
    cfg = CONFIGS[cfg_id]
    assert isinstance(cfg, PrefillConfig)
    return make_prefill_inputs(draw_lengths(cfg), cfg.H, cfg.D, cfg.D, cfg.dtype,
                               cfg.g_mean, cfg.s0_std, cfg.seed, heads=heads)


def make_decode_state(N: int, H: int, dk: int, dv: int, s0_std: float, seed: int,
                      heads: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Initial decode state [N, Hs, dk, dv] fp32 ~ N(0, s0_std^2), per-head streams."""
    heads = list(range(H)) if heads is None else list(heads)
    S = torch.empty(N, len(heads), dk, dv, dtype=torch.float32)
    for j, h in enumerate(heads):
        gen = _head_generator(seed + 17, h)
        S[:, j] = s0_std * torch.randn(N, dk, dv, generator=gen)
    return S


def make_decode_step_inputs(N: int, H: int, dk: int, dv: int, dtype: torch.dtype,
                            g_mean: float, seed: int, step: int,
                            heads: Optional[Sequence[int]] = None) -> dict:
    """Fresh one-token inputs for decode step `step`: q, k [N, Hs, dk], v [N, Hs, dv],
    g [N, Hs, dk] fp32, beta [N, Hs] fp32 (same recipe as prefill, one token per sequence)."""
    d = make_prefill_inputs([1] * N, H, dk, dv, dtype, g_mean, 0.0,
                            seed + STEP_SEED_STRIDE * (step + 1), heads=heads)
    return dict(q=d["q"], k=d["k"], v=d["v"], g=d["g"], beta=d["beta"])


def make_prefill_inputs_device(lengths: Sequence[int], H: int, dk: int, dv: int,
                               dtype: torch.dtype, g_mean: float, s0_std: float, seed: int,
                               cpu_heads: Sequence[int] = (), device="cuda") -> dict:
    """Large batches: draw every head with a seeded torch device generator (same recipe),
    except `cpu_heads`, which are drawn from their per-head CPU streams exactly as
    make_prefill_inputs does (so an oracle can be given those heads' identical bytes).
    Returns device tensors plus `cpu` = the make_prefill_inputs(..., heads=cpu_heads) dict."""
    T = int(sum(lengths))
    N = len(lengths)
    gen = torch.Generator(device=device).manual_seed(seed)
    q = torch.empty(T, H, dk, dtype=dtype, device=device)
    k = torch.empty(T, H, dk, dtype=dtype, device=device)
    v = torch.empty(T, H, dv, dtype=dtype, device=device)
    g = torch.empty(T, H, dk, dtype=torch.float32, device=device)
    beta = torch.empty(T, H, dtype=torch.float32, device=device)
    s0 = torch.empty(N, H, dk, dv, dtype=torch.float32, device=device) if s0_std > 0 else None
    for h in range(H):
        q[:, h] = _l2_normalise(torch.randn(T, dk, generator=gen, device=device)).to(dtype)
        k[:, h] = _l2_normalise(torch.randn(T, dk, generator=gen, device=device)).to(dtype)
        v[:, h] = torch.randn(T, dv, generator=gen, device=device).to(dtype)
        beta[:, h] = torch.sigmoid(torch.randn(T, generator=gen, device=device))
        g[:, h] = torch.nn.functional.logsigmoid(
            g_mean + torch.randn(T, dk, generator=gen, device=device))
        if s0 is not None:
            s0[:, h] = s0_std * torch.randn(N, dk, dv, generator=gen, device=device)
    cpu = make_prefill_inputs(lengths, H, dk, dv, dtype, g_mean, s0_std, seed, heads=cpu_heads)
    for j, h in enumerate(cpu_heads):
        for key, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta)):
            t[:, h] = cpu[key][:, j].to(device)
        if s0 is not None:
            s0[:, h] = cpu["s0"][:, j].to(device)
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu_seqlens_of(lengths).to(device),
                s0=s0, cpu=cpu)


def make_raw_prefill_inputs(lengths: Sequence[int], H: int, dk: int, dv: int, dtype: torch.dtype,
                            g_mean: float, s0_std: float, seed: int, scalar_gate: bool = False) -> dict:
    """Inputs as the layer hands them over before its elementwise prologue: q, k ~ N(0, 1)
    not normalised (cast to `dtype`), v ~ N(0, 1); gate logits ~ N(g_mean, 1) fp32 [T, H, dk]
    (or [T, H] with scalar_gate); beta logits ~ N(0, 1) fp32 [T, H]; initial state as in
    make_prefill_inputs.  One seeded CPU generator per head, in the order q, k, v,
    beta-logits, gate-logits, initial state."""
    T = int(sum(lengths))
    N = len(lengths)
    q = torch.empty(T, H, dk, dtype=dtype)
    k = torch.empty(T, H, dk, dtype=dtype)
    v = torch.empty(T, H, dv, dtype=dtype)
    g = torch.empty((T, H) if scalar_gate else (T, H, dk), dtype=torch.float32)
    beta = torch.empty(T, H, dtype=torch.float32)
    s0 = torch.empty(N, H, dk, dv, dtype=torch.float32) if s0_std > 0 else None
    for h in range(H):
        gen = _head_generator(seed, h)
        q[:, h] = torch.randn(T, dk, generator=gen).to(dtype)
        k[:, h] = torch.randn(T, dk, generator=gen).to(dtype)
        v[:, h] = torch.randn(T, dv, generator=gen).to(dtype)
        beta[:, h] = torch.randn(T, generator=gen)
        g[:, h] = g_mean + torch.randn(*((T,) if scalar_gate else (T, dk)), generator=gen)
        if s0 is not None:
            s0[:, h] = s0_std * torch.randn(N, dk, dv, generator=gen)
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu_seqlens_of(lengths), s0=s0)
