#!/usr/bin/env python
"""KDA benchmark: prefill tokens/s (H=32, D=128) + decode state GB/s, as % of roofline.

One JSON line on rank 0.  The timed "step" is one call of the whole prefill path
(kda_prefill: chunking, cumulative decay, decayed operands, L / Aqk, UT transform,
pseudo-values, chunk recurrence, final state) on the single-sequence workload
B=1, H=32, T=8192, D=128, C=64, bf16 inputs, inputs resident in HBM.  The decode step
(N=256 x H=32, D=128, 64 consecutive in-place steps) is timed in the same run and
reported under "decode".  Multi-GPU runs are independent replicas (every rank owns its
own problem; there is no exchange on the path), so scaling is weak and the job value
is the sum of tokens over ranks divided by the slowest rank's time.

--impl reference runs the fp64 CPU oracle instead (bounded samples of the same
workload on the host cores); under torchrun only rank 0 does, the others exit.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H=32,D=128) + decode state GB/s, as % of B200 roofline"
PREFILL_CFG = 1
DECODE_CFG = 3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- host logic
def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own independent problem of the same shape."""
    return base_seed + 104_729 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def prefill_page_counts(lengths, H, D, C):
    """The pages' per-chunk-head counts (FlashKDA section): 12C^3 + 8C^2 D + 6 C D^2 FLOPs
    and 8C^2 + 22 C D bytes per chunk per head, plus 8 D^2 bytes of state per head.
    A partial chunk counts as a whole chunk."""
    chunks = sum((n + C - 1) // C for n in lengths)
    ch = chunks * H
    flops = ch * (12 * C ** 3 + 8 * C * C * D + 6 * C * D * D)
    bytes_ = ch * (8 * C * C + 22 * C * D) + 8 * D * D * len(lengths) * H
    return flops, bytes_


def prefill_stage_page_bytes(lengths, H, D, C):
    """The pages' byte count split by stage (FlashKDA section): the preparation reads
    q, k, v (3 x 2CD) and writes the chunk tensors (3 x 2CD + 2 x 2C^2); the recurrence
    reads them back and writes O (2 x 2CD), plus the 8 D^2 state bytes per head."""
    chunks = sum((n + C - 1) // C for n in lengths)
    ch = chunks * H
    prep = ch * (3 * 2 * C * D + 3 * 2 * C * D + 2 * 2 * C * C)
    rest = ch * (3 * 2 * C * D + 2 * 2 * C * C + 2 * 2 * C * D) + 8 * D * D * len(lengths) * H
    return prep, rest


# CUDA sources each kernel's recorded counters depend on (its own file and the helpers it uses)
KERNEL_SOURCES = {
    "prep_kernel": ("kda_common.cuh", "kda_sm100.cuh", "kda_prefill_tc.cuh",
                    "kda_prep_strong.cuh", "kda_chunk_simt.cuh"),
    "rec_kernel": ("kda_common.cuh", "kda_sm100.cuh", "kda_prefill_tc.cuh",
                   "kda_prep_strong.cuh", "kda_chunk_simt.cuh"),
    "decode_kernel": ("kda_common.cuh", "kda_decode.cuh"),
}


def source_digest(files=None):
    """Short hash of the CUDA sources (all of csrc, or the named files), to tell whether
    recorded ncu counters still apply."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_rule_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` recorded from an ncu capture in profiles/
    ('<kernel> traffic_bytes_per_launch <N> sources <digest>'), or None when absent or
    taken on different sources of that kernel (KERNEL_SOURCES)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as fh:
            for line in fh:
                f = line.split()
                if len(f) >= 5 and f[0] == kernel and f[1] == "traffic_bytes_per_launch":
                    return int(f[2]) if f[4] == source_digest(KERNEL_SOURCES.get(kernel)) else None
    except OSError:
        pass
    return None


def prefill_strict_bytes(lengths, H, D, in_bytes, has_s0, has_final):
    """Bytes the method itself must move: q, k, v, out in the input dtype, g fp32 (dk per
    token-head), beta fp32, and the fp32 states read/written."""
    T = sum(lengths)
    per_tok_head = 4 * D * in_bytes + 4 * D + 4
    states = 4 * D * D * len(lengths) * H * ((1 if has_s0 else 0) + (1 if has_final else 0))
    return T * H * per_tok_head + states


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a background thread."""
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device, period_s: float = 0.0002):
        self.period = period_s
        self.samples, self.max_mhz, self.ok = [], None, False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            p = torch.cuda.get_device_properties(device)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML unavailable: report no clocks
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            # a short GIL switch interval, so that the sampling thread runs while the main
            # thread issues launches (the default 5 ms left a few-ms region with one sample)
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(self.period / 2)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            # the thread is sampling before the region starts (its start-up took a few ms,
            # longer than a short timed region); what it took before then is dropped
            t0 = time.perf_counter()
            while len(self.samples) < 2 and time.perf_counter() - t0 < 1.0:
                time.sleep(self.period)
            del self.samples[:]
        return self

    def __exit__(self, *exc):
        if self.ok:
            sys.setswitchinterval(self._switch)
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample_tokens_per_s(inp, target_s: float):
    """Time the fp64 oracle on the first Ts tokens (all heads) of the prefill workload,
    Ts sized for about `target_s` seconds.  Returns (tokens/s, Ts, seconds, threads)."""
    import oracle
    T = inp["q"].shape[0]
    H = inp["q"].shape[1]
    threads = min(oracle.default_threads(), H)

    def run(ts):
        t0 = time.perf_counter()
        oracle.prefill(inp["q"][:ts], inp["k"][:ts], inp["v"][:ts], inp["g"][:ts],
                       inp["beta"][:ts], [0, ts], nthreads=threads)
        return time.perf_counter() - t0

    ts = 32
    dt = run(ts)
    ts = int(max(32, min(T, ts * target_s / max(dt, 1e-6))))
    dt = run(ts)
    reps, total = 1, dt
    while total < target_s * 0.8 and reps < 1000:   # whole workload is quick: repeat it
        total += run(ts)
        reps += 1
    return reps * ts / total, ts, total, threads


# ----------------------------------------------------------------------------- GPU arm
def timed(stream, dev, world, steps, fn):
    """Run fn `steps` times between CUDA events on `stream` (barrier + synchronize on
    both sides); returns (this rank's ms per step, max over ranks, clock summary)."""
    import torch
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms_local = e0.elapsed_time(e1) / steps
    return ms_local, max_over_ranks(ms_local, world, dev), clk.summary()


def setup_prefill(dev, rank, cfg_id=PREFILL_CFG):
    import torch
    from linear_attention_rule_b200 import kda, synthetic
    cfg = synthetic.CONFIGS[cfg_id]
    lengths = synthetic.draw_lengths(cfg)
    D, H, C = cfg.D, cfg.H, cfg.C
    if sum(lengths) * H > (1 << 22):   # large batches are drawn on the device (same recipe)
        d = synthetic.make_prefill_inputs_device(lengths, H, D, D, cfg.dtype, cfg.g_mean,
                                                 cfg.s0_std, rank_seed(cfg.seed, rank), device=dev)
        d.pop("cpu")
        inp = None
    else:
        inp = synthetic.make_prefill_inputs(lengths, H, D, D, cfg.dtype, cfg.g_mean, cfg.s0_std,
                                            rank_seed(cfg.seed, rank))
        d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    T, N = sum(lengths), len(lengths)
    out = torch.empty(T, H, D, dtype=cfg.dtype, device=dev)
    fin = torch.empty(N, H, D, D, dtype=torch.float32, device=dev)
    ws_bytes = kda.kda_prefill_workspace_size(T, N, H, D, D, C, cfg.dtype)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    return dict(cfg=cfg, lengths=lengths, inp=inp, d=d, out=out, fin=fin, ws=ws, T=T, N=N,
                D=D, H=H, C=C)


def bench_prefill(args, P, dev, stream, world, peaks):
    import torch
    from linear_attention_rule_b200 import kda
    cfg, d, D, H, C, T = P["cfg"], P["d"], P["D"], P["H"], P["C"], P["T"]

    def step():
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], P["out"],
                        initial_state=d["s0"], final_state=P["fin"], C=C, workspace=P["ws"],
                        stream=stream)

    for _ in range(args.warmup):
        step()
    assert kda.kda_get_device_status(stream) == kda.KDA_OK
    ms_local, ms, clocks = timed(stream, dev, world, args.steps, step)
    assert kda.kda_get_device_status(stream) == kda.KDA_OK
    flops, page_bytes = prefill_page_counts(P["lengths"], H, D, C)
    strict = prefill_strict_bytes(P["lengths"], H, D, 2 if cfg.dtype.itemsize == 2 else 4,
                                  d["s0"] is not None, True)
    t_s = ms_local * 1e-3
    res = dict(value=world * T / (ms * 1e-3), ms=ms, ms_local=ms_local, clocks=clocks,
               launches=kda.kda_prefill_launches(T, P["N"], H, D, D, C, cfg.dtype) * args.steps, step=step,
               whole_frac=page_bytes / t_s / 1e9 / peaks["hbm_gbs"],
               tensor_frac=flops / t_s / 1e12 / peaks["bf16_tflops"],
               strict_frac=strict / t_s / 1e9 / peaks["hbm_gbs"])

    # Per kernel: the same work through the staged entry points, CUDA events between the
    # stages on the launching stream.
    stage_ms = None
    if kda.tensor_core_path(cfg.dtype, D):
        ws = P["ws"]
        stages = [
            ("prep_kernel", lambda: kda.kda_prefill_prepare(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                                            d["cu_seqlens"], ws, C=C, stream=stream)),
            ("rec_kernel", lambda: kda.kda_prefill_scan(P["out"], d["cu_seqlens"], ws,
                                                        initial_state=d["s0"], final_state=P["fin"],
                                                        C=C, stream=stream)),
        ]
        for _ in range(args.warmup):
            for _, f in stages:
                f()
        torch.cuda.synchronize(dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
              for _ in range(args.steps)]
        for i in range(args.steps):
            ev[i][0].record(stream)
            for j, (_, f) in enumerate(stages):
                f()
                ev[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
        assert kda.kda_get_device_status(stream) == kda.KDA_OK
        stage_ms = {name: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)) / args.steps
                    for j, (name, _) in enumerate(stages)}
        prep_bytes, _ = prefill_stage_page_bytes(P["lengths"], H, D, C)
        top = max(stage_ms, key=stage_ms.get)
        per_launch = {"prep_kernel": prep_bytes}
        if top in per_launch:
            achieved = per_launch[top] / (stage_ms[top] * 1e-3) / 1e9
            res["roofline"] = {
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": recorded_traffic(top), "kernel": "kda::tc::" + top,
                "bytes_per_launch": per_launch[top],
                "counts": "pages' preparation bytes 3x2CD + (3x2CD + 2x2C^2) per chunk-head",
                "peak_source": peaks["source"], "ms_per_launch": round(stage_ms[top], 4),
            }
        res["stage_ms"] = {k: round(v, 4) for k, v in stage_ms.items()}
    if "roofline" not in res:
        achieved = page_bytes / t_s / 1e9
        res["roofline"] = {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
            "kernel": "kda_prefill (single kernel)", "bytes_per_launch": page_bytes,
            "counts": "pages' 8C^2+22CD bytes per chunk-head + 8D^2 per head",
            "peak_source": peaks["source"],
        }
    res["roofline"]["path_frac"] = round(res["whole_frac"], 4)
    res["roofline"]["path_strict_frac"] = round(res["strict_frac"], 4)
    res["roofline"]["path_tensor_frac"] = round(res["tensor_frac"], 4)
    return res


def bench_decode(args, dev, stream, rank, world, peaks):
    import torch
    from linear_attention_rule_b200 import kda, synthetic
    dcfg = synthetic.CONFIGS[DECODE_CFG]
    Nd, Hd, Dd = dcfg.N, dcfg.H, dcfg.D
    S = synthetic.make_decode_state(Nd, Hd, Dd, Dd, dcfg.s0_std, rank_seed(dcfg.seed, rank)).to(dev)
    steps_in = []
    for s in range(dcfg.steps):
        x = synthetic.make_decode_step_inputs(Nd, Hd, Dd, Dd, dcfg.dtype, dcfg.g_mean,
                                              rank_seed(dcfg.seed, rank), s)
        steps_in.append({k: v.to(dev) for k, v in x.items()})
    dout = torch.empty(Nd, Hd, Dd, dtype=dcfg.dtype, device=dev)

    def step():
        for x in steps_in:
            kda.kda_decode(x["q"], x["k"], x["v"], x["g"], x["beta"], S, dout, stream=stream)

    for _ in range(args.warmup):
        step()
    ms_local, ms, clocks = timed(stream, dev, world, args.steps, step)
    state_bytes = 8 * Dd * Dd * Nd * Hd * dcfg.steps
    gbs_local = state_bytes / (ms_local * 1e-3) / 1e9
    return {
        "workload": dcfg.name, "value": round(world * state_bytes / (ms * 1e-3) / 1e9, 1),
        "unit": "GB/s (fp32 state read+write)", "ms_per_step": round(ms, 4),
        "steps_per_call": dcfg.steps,
        "seq_tokens_per_s": round(world * Nd * dcfg.steps / (ms * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(gbs_local, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(gbs_local / peaks["hbm_gbs"], 4),
                     "traffic": recorded_traffic("decode_kernel"), "kernel": "kda::decode_kernel",
                     "bytes_per_launch": 8 * Dd * Dd * Nd * Hd,
                     "counts": "pages' 8 D^2 bytes per head-token", "peak_source": peaks["source"]},
        "clocks": clocks, "gpu_launches": dcfg.steps * args.steps,
    }


def bench_e2e(args, P, pre, dev, stream, world):
    """Same metric through the public API with host buffers: every step copies its inputs
    from pinned host memory to the device, runs the prefill and copies O and the final
    state back, all inside the timed region.  Steps are pipelined the way a serving loop
    would run them: the read-back of step i (on a second stream, from one of two output
    buffers) overlaps the upload of step i+1 (two input buffers), so the two PCIe
    directions run at the same time."""
    import torch
    from linear_attention_rule_b200 import kda
    inp, C = P["inp"], P["C"]
    h = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    keys = ("q", "k", "v", "g", "beta", "cu_seqlens") + (("s0",) if inp["s0"] is not None else ())
    dbuf = [P["d"], {k: (P["d"][k].clone() if P["d"][k] is not None else None) for k in P["d"]}]
    obuf = [(P["out"], P["fin"]), (torch.empty_like(P["out"]), torch.empty_like(P["fin"]))]
    hout = [torch.empty_like(P["out"], device="cpu").pin_memory() for _ in range(2)]
    hfin = [torch.empty_like(P["fin"], device="cpu").pin_memory() for _ in range(2)]
    back = torch.cuda.Stream(dev)
    done = [torch.cuda.Event() for _ in range(2)]    # prefill i done (on `stream`)
    freed = [None, None]                              # read-back of the buffer's last step done
    counter = [0]

    def step():
        i = counter[0]
        counter[0] += 1
        b = i & 1
        d, (out, fin) = dbuf[b], obuf[b]
        for k in keys:
            d[k].copy_(h[k], non_blocking=True)
        if freed[b] is not None:
            stream.wait_event(freed[b])              # out / fin of step i-2 have been read back
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                        initial_state=d["s0"], final_state=fin, C=C, workspace=P["ws"], stream=stream)
        done[b].record(stream)
        back.wait_event(done[b])
        with torch.cuda.stream(back):
            hout[b].copy_(out, non_blocking=True)
            hfin[b].copy_(fin, non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(back)
        freed[b] = ev

    def run(n):
        for _ in range(n):
            step()
        stream.wait_stream(back)                      # the last read-back inside the region

    run(args.warmup)
    _, ms, _ = timed(stream, dev, world, 1, lambda: run(args.steps))
    ms /= args.steps
    h2d = sum(h[k].numel() * h[k].element_size() for k in keys)
    d2h = hout[0].numel() * hout[0].element_size() + hfin[0].numel() * hfin[0].element_size()
    return {"value": round(world * P["T"] / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4),
            "pipelined": "read-back of step i overlaps upload of step i+1"}


def bench_crossover(args, dev, stream):
    """Serial chains vs the chunk-parallel scan of the recurrence: kda_prefill_ex with and
    without KDA_IN_SERIAL_CHAINS (the preparation is the same in both) on one long sequence
    for a grid of (H, T); inputs drawn on the device."""
    import torch
    from linear_attention_rule_b200 import kda, synthetic
    rows = []
    for H, T in [(2, 1 << 18), (2, 1 << 20), (4, 1 << 16), (4, 1 << 18), (4, 1 << 20), (8, 1 << 16),
                 (8, 1 << 18), (8, 1 << 20), (16, 1 << 15), (16, 1 << 18), (32, 8192), (32, 1 << 15),
                 (32, 1 << 18)]:
        d = synthetic.make_prefill_inputs_device([T], H, 128, 128, torch.bfloat16, 3.0, 0.0, 77, device=dev)
        d.pop("cpu")
        out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
        fin = torch.empty(1, H, 128, 128, device=dev)
        ws = torch.empty(kda.kda_prefill_workspace_size(T, 1, H, 128, 128, 64, torch.bfloat16),
                         dtype=torch.uint8, device=dev)
        res = {}
        for name, flags in (("serial", kda.KDA_IN_SERIAL_CHAINS), ("auto", 0)):
            def step():
                kda.kda_prefill_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, flags,
                                   final_state=fin, workspace=ws, stream=stream)
            for _ in range(args.warmup):
                step()
            steps = max(2, min(args.steps, int(2e7 // (T * H)) + 2))
            ms, _, _ = timed(stream, dev, 1, steps, step)
            assert kda.kda_get_device_status(stream) == kda.KDA_OK
            res[name] = round(ms, 4)
        rows.append({"H": H, "T": T, "serial_ms": res["serial"], "auto_ms": res["auto"],
                     "speedup": round(res["serial"] / res["auto"], 3)})
        del d, out, fin, ws
        torch.cuda.empty_cache()
    return {"crossover": rows}


def bench_windows(args, dev, stream):
    """The cost of a bounded workspace: the prefill of configs 1 and 4 with workspaces from
    the full size down to the allocation-free scratch (64 MiB), the chunks then running in
    windows (kda_prefill_windows); bitwise the same results."""
    import torch
    from linear_attention_rule_b200 import kda
    rows = []
    for cfg_id in (1, 4):
        P = setup_prefill(dev, 0, cfg_id)
        d, T, N, H, D, C = P["d"], P["T"], P["N"], P["H"], P["D"], P["C"]
        full = kda.kda_prefill_workspace_size(T, N, H, D, D, C, P["cfg"].dtype)
        budgets = [full, 4 << 30, 1 << 30, 256 << 20, kda.NOALLOC_SCRATCH_BYTES]
        P["ws"] = None
        torch.cuda.empty_cache()
        ws = torch.empty(full, dtype=torch.uint8, device=dev)
        for b in budgets:
            if b > full:
                continue
            n = kda.kda_prefill_windows(T, N, H, D, D, C, P["cfg"].dtype, b)
            view = ws[:b]

            def step():
                kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], P["out"],
                                initial_state=d["s0"], final_state=P["fin"], C=C, workspace=view, stream=stream)
            for _ in range(args.warmup):
                step()
            steps = max(2, min(args.steps, int(2e7 // T) + 2))
            ms, _, _ = timed(stream, dev, 1, steps, step)
            assert kda.kda_get_device_status(stream) == kda.KDA_OK
            rows.append({"workload": P["cfg"].name, "workspace_bytes": b, "windows": n, "ms": round(ms, 4),
                         "tokens_per_s": round(T / (ms * 1e-3), 1)})
        del P, ws, view
        torch.cuda.empty_cache()
    return {"windows": rows}


def bench_d64(args, dev, stream):
    """bf16 with d = 64 (the tensor-core kernels on the first 64 channels of a 128-channel
    problem) against d = 128 on the same shape: T = 8,192 tokens, H = 32 and 64 heads."""
    import torch
    from linear_attention_rule_b200 import kda, synthetic
    rows = []
    for D, H in ((128, 32), (64, 32), (64, 64)):
        T = 8192
        d = synthetic.make_prefill_inputs_device([T], H, D, D, torch.bfloat16, 3.0, 0.0, 5, device=dev)
        d.pop("cpu")
        out = torch.empty(T, H, D, dtype=torch.bfloat16, device=dev)
        fin = torch.empty(1, H, D, D, device=dev)
        ws = torch.empty(kda.kda_prefill_workspace_size(T, 1, H, D, D, 64, torch.bfloat16), dtype=torch.uint8,
                         device=dev)

        def step():
            kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, final_state=fin,
                            workspace=ws, stream=stream)
        for _ in range(args.warmup):
            step()
        ms, _, _ = timed(stream, dev, 1, args.steps, step)
        assert kda.kda_get_device_status(stream) == kda.KDA_OK
        rows.append({"D": D, "H": H, "T": T, "ms": round(ms, 4), "tokens_per_s": round(T / (ms * 1e-3), 1)})
        del d, out, fin, ws
        torch.cuda.empty_cache()
    return {"d64": rows}


def bench_gpu(args):
    import torch
    from linear_attention_rule_b200 import kda

    rank, local_rank, world = rank_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)

    def prefill_config_entry(cfg_id):
        """Another prefill configuration of the metric (few steps): tokens/s, the dominant
        kernel's roofline and the path fractions, stage times and clocks."""
        import argparse as _ap
        sub = _ap.Namespace(**vars(args))
        sub.steps = min(args.steps, 5)
        P = setup_prefill(dev, rank, cfg_id)
        pre = bench_prefill(sub, P, dev, stream, world, peaks)
        entry = {"workload": P["cfg"].name, "T": P["T"], "num_seqs": P["N"],
                 "value": round(pre["value"], 1), "unit": "tokens/s", "steps": sub.steps,
                 "warmup": sub.warmup, "ms_per_step": round(pre["ms"], 4),
                 "roofline": pre["roofline"], "stage_ms": pre.get("stage_ms"),
                 "clocks": pre["clocks"], "gpu_launches": pre["launches"]}
        del P, pre
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        return entry

    line = {}
    if args.workload == "crossover":
        line = bench_crossover(args, dev, stream)
    elif args.workload == "windows":
        line = bench_windows(args, dev, stream)
    elif args.workload == "d64":
        line = bench_d64(args, dev, stream)
    elif args.workload in ("config2", "config4"):
        P = setup_prefill(dev, rank, int(args.workload[-1]))
        pre = bench_prefill(args, P, dev, stream, world, peaks)
        line = {"workload": P["cfg"].name, "value": round(pre["value"], 1), "unit": "tokens/s",
                "ms_per_step": round(pre["ms"], 4), "roofline": pre["roofline"],
                "stage_ms": pre.get("stage_ms"), "clocks": pre["clocks"], "n_gpus": world}
    elif args.workload in ("all", "prefill"):
        P = setup_prefill(dev, rank)
        pre = bench_prefill(args, P, dev, stream, world, peaks)
        decode = bench_decode(args, dev, stream, rank, world, peaks) if args.workload == "all" else None
        e2e = None if args.no_e2e else bench_e2e(args, P, pre, dev, stream, world)
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline and P["inp"] is not None:
            tps, ts, secs, threads = oracle_sample_tokens_per_s(P["inp"], args.cpu_seconds)
            cpu = {"value": round(tps, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                   "sample": "first %d tokens x all %d heads of the same workload (repeated), "
                             "fp64, %.1f s" % (ts, P["H"], secs)}
        cfg = P["cfg"]
        line = {
            "metric": METRIC, "value": round(pre["value"], 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(pre["ms"], 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": kda.prefill_compute_dtype(cfg.dtype, P["D"]),
            "data": "synthetic",
            "config": prefill_config_dict(cfg, P["T"], P["d"], world),
            "roofline": pre["roofline"], "stage_ms": pre.get("stage_ms"), "decode": decode,
            "e2e": e2e, "cpu_baseline": cpu, "clocks": pre["clocks"],
            "gpu_launches": pre["launches"],
        }
        if args.workload == "all" and not args.no_extra_configs:
            del P, pre
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
            line["prefill_configs"] = {"config2": prefill_config_entry(2),
                                       "config4": prefill_config_entry(4)}
    else:
        line = {"decode": bench_decode(args, dev, stream, rank, world, peaks)}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def prefill_config_dict(cfg, T, tensors, world):
    """The prefill workload's config, the same for both arms (the input bytes from the
    tensors of either arm: the same shapes and dtypes)."""
    nbytes = sum(tensors[k].numel() * tensors[k].element_size() for k in ("q", "k", "v", "g", "beta"))
    return {"workload": cfg.name, "T": T, "H": cfg.H, "D": cfg.D, "C": cfg.C,
            "l2": "inputs larger than L2 (%.0f MB resident per step)" % (nbytes / 1e6),
            "parallelism": "replicas" if world > 1 else "single GPU"}


# ----------------------------------------------------------------------------- reference arm
def bench_reference(args):
    rank, _, world = rank_env()
    if rank != 0:
        return
    import oracle
    from linear_attention_rule_b200 import synthetic
    cfg = synthetic.CONFIGS[PREFILL_CFG]
    lengths = synthetic.draw_lengths(cfg)
    inp = synthetic.make_prefill_inputs(lengths, cfg.H, cfg.D, cfg.D, cfg.dtype, cfg.g_mean,
                                        cfg.s0_std, cfg.seed)
    H = cfg.H
    threads = min(oracle.default_threads(), H)
    # size one step for about args.cpu_seconds / 2 of fp64 work, less when many steps are
    # asked for, so that warm-up and timed steps together take about 90 s at most
    per_step = max(0.05, min(args.cpu_seconds / 2, 90.0 / (args.steps + args.warmup)))
    _, ts, _, _ = oracle_sample_tokens_per_s(inp, per_step)

    def step():
        oracle.prefill(inp["q"][:ts], inp["k"][:ts], inp["v"][:ts], inp["g"][:ts],
                       inp["beta"][:ts], [0, ts], nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = (time.perf_counter() - t0) / args.steps
    value = ts / secs
    sample = "first %d tokens x all %d heads of %s per step, fp64 oracle" % (ts, H, cfg.name)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": prefill_config_dict(cfg, sum(lengths), inp, world),
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the varlen (config 2) and long-context (config 4) prefill entries")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--workload", choices=["all", "prefill", "decode", "config2", "config4", "crossover", "windows", "d64"],
                    default="all",
                    help="restrict the run (profiling) or measure another prefill config; "
                         "the driver's JSON line is 'all'")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    _, _, world = rank_env()
    if world != args.gpus:
        print("note: --gpus %d but WORLD_SIZE %d; using WORLD_SIZE" % (args.gpus, world),
              file=sys.stderr)
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_gpu(args)


if __name__ == "__main__":
    main()
