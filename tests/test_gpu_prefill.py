"""GPU parity of kda_prefill against the fp64 oracle, through the C-ABI."""
import numpy as np
import pytest
import torch

from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import TOL, check_prefill, run_prefill, to_device

pytestmark = pytest.mark.gpu


def _inputs(lens, H, D, dtype, s0_std=0.02, seed=5, g_mean=3.0):
    return synthetic.make_prefill_inputs(lens, H, D, D, dtype, g_mean, s0_std, seed)


def test_config0_tiny_fp32():
    """Config 0: B=1, H=2, T=256, D=64, C=64, fp32, zero initial state; tolerance 1e-4."""
    inp = synthetic.make_config_inputs(0)
    out, fin = run_prefill(inp, C=64)
    e_o, e_f = check_prefill(inp, out, fin, tol=1e-4)
    print("config0 max rel err out %.3g final %.3g" % (e_o, e_f))


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_fp32_ragged_chunks(C, D):
    """fp32: lengths around the chunk size (1, C-1, C, C+1, several chunks + tail, empty)."""
    lens = [1, C - 1, C, C + 1, 0, 5 * C + 3]
    inp = _inputs(lens, 3, D, torch.float32, seed=C + D)
    out, fin = run_prefill(inp, C=C)
    check_prefill(inp, out, fin, tol=1e-4)


def test_bf16_ragged_varlen_small():
    lens = [1000, 64, 63, 65, 1, 0, 300]
    inp = _inputs(lens, 4, 128, torch.bfloat16, seed=11)
    out, fin = run_prefill(inp, C=64)
    check_prefill(inp, out, fin, chunk=64)


def test_bf16_many_sequence_heads():
    """More (sequence, head) pairs than the recurrence can run at once on the SMs (192 CTAs),
    ragged and empty sequences included."""
    lens = [100, 64, 1, 300, 0, 129]
    inp = _inputs(lens, 32, 128, torch.bfloat16, seed=13)
    out, fin = run_prefill(inp, C=64)
    check_prefill(inp, out, fin, heads=[0, 7, 31])


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 64),
                                     (torch.float32, 128)])
@pytest.mark.parametrize("g_mean", [-3.0, -8.0])
def test_strong_decay_by_default(dtype, D, g_mean):
    """Gates logsigmoid(N(-3, 1)) (a full chunk's log-decay near -190 per channel, so e^{-a}
    alone would overflow fp32 and bf16) and logsigmoid(N(-8, 1)) (near -8 per token: even 16
    tokens pass -88), with no flag: every path matches the oracle."""
    inp = _inputs([200, 64, 70, 1], 2, D, dtype, seed=17, g_mean=g_mean)
    assert float(inp["g"][:64].sum(0).max()) < -150      # the premise: far beyond e^{88}
    out, fin = run_prefill(inp, C=64)
    check_prefill(inp, out, fin, chunk=64)


def test_strong_and_mild_chunks_in_one_call():
    """Sequences whose chunks take the tensor-core preparation and sequences whose chunks are
    too strongly decayed for it, packed together (and one chunk with a single strong channel
    among mild ones): the records of both preparations meet in one recurrence."""
    lens = [300, 130, 64, 200]
    inp = _inputs(lens, 3, 128, torch.bfloat16, seed=71, g_mean=3.0)
    strong = _inputs(lens, 3, 128, torch.bfloat16, seed=72, g_mean=-4.0)
    cu = inp["cu_seqlens"].tolist()
    inp["g"][cu[1]:cu[2]] = strong["g"][cu[1]:cu[2]]          # sequence 1 strong everywhere
    inp["g"][cu[3] + 64:cu[3] + 128, 1, 5] = -3.0              # one channel of one chunk of head 1
    out, fin = run_prefill(inp, C=64)
    check_prefill(inp, out, fin, chunk=64)


def test_strong_decay_with_prologue_and_scalar_gate():
    """Strong decay through the Gated DeltaNet scalar gate and through gate logits."""
    import oracle
    lens = [150, 64]
    inp = _inputs(lens, 2, 128, torch.bfloat16, seed=73, g_mean=-4.0)
    gs = inp["g"][:, :, 0].contiguous()                        # one gate per (token, head)
    d = to_device(inp)
    out = torch.full_like(d["v"], float("nan"))
    fin = torch.full((2, 2, 128, 128), float("nan"), device="cuda")
    kda.kda_prefill_gdn(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], d["cu_seqlens"], out,
                        initial_state=d["s0"], final_state=fin)
    assert kda.kda_get_device_status() == kda.KDA_OK
    g_full = gs[..., None].expand(-1, -1, 128).contiguous()
    o_ref, f_ref = oracle.prefill(inp["q"], inp["k"], inp["v"], g_full, inp["beta"], inp["cu_seqlens"],
                                  s0=inp["s0"])
    tol = TOL[torch.bfloat16]
    assert oracle.max_rel_frobenius_per_slice(out.double().cpu().numpy(), o_ref, inp["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin.double().cpu().numpy(), f_ref) <= tol
    # gate logits N(-3, 1): logsigmoid applied inside, strong decay in every chunk
    logits = -3.0 + torch.randn(inp["g"].shape, generator=torch.Generator().manual_seed(74))
    out2 = torch.full_like(d["v"], float("nan"))
    kda.kda_prefill_ex(d["q"], d["k"], d["v"], logits.cuda(), d["beta"], d["cu_seqlens"], out2,
                       kda.KDA_IN_G_LOGITS, initial_state=d["s0"], final_state=fin)
    assert kda.kda_get_device_status() == kda.KDA_OK
    g2 = torch.from_numpy(oracle.logsigmoid(logits)).float()
    o_ref2, f_ref2 = oracle.prefill(inp["q"], inp["k"], inp["v"], g2, inp["beta"], inp["cu_seqlens"],
                                    s0=inp["s0"])
    assert oracle.max_rel_frobenius_per_slice(out2.double().cpu().numpy(), o_ref2, inp["cu_seqlens"]) <= tol
    assert oracle.max_rel_frobenius_states(fin.double().cpu().numpy(), f_ref2) <= tol


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_strong_decay_flag_is_bit_identical_on_mild_decay(dtype, D):
    """KDA_IN_STRONG_DECAY is accepted and ignored: results are the same bit for bit."""
    inp = _inputs([300, 64, 1, 129], 3, D, dtype, seed=19, g_mean=3.0)
    assert float(inp["g"][:64].sum(0).min()) > -64
    o0, f0 = run_prefill(inp, C=64)
    o1, f1 = run_prefill(inp, C=64, in_flags=kda.KDA_IN_STRONG_DECAY)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(f0, f1)


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_degenerate_beta_zero_is_pure_channel_decay(dtype, D):
    """beta = 0 writes nothing: the state only decays channel-wise, S_T = diag(e^{sum g}) S_0
    (closed form, checked directly in fp64), and every output is read from it."""
    lens = [200, 64, 7]
    inp = _inputs(lens, 2, D, dtype, seed=23)
    inp["beta"].zero_()
    out, fin = run_prefill(inp)
    check_prefill(inp, out, fin)
    cu = inp["cu_seqlens"].tolist()
    g = inp["g"].double().numpy()
    s0 = inp["s0"].double().numpy()
    import oracle
    for n in range(len(lens)):
        decay = np.exp(g[cu[n]:cu[n + 1]].sum(0))          # [H, dk]
        ref = decay[:, :, None] * s0[n]
        assert oracle.max_rel_frobenius_states(fin[n:n + 1], ref[None]) <= TOL[dtype]


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_degenerate_no_decay_is_the_delta_rule(dtype, D):
    """g = 0 (alpha = 1): the plain delta rule, no forgetting over 300 tokens."""
    inp = _inputs([300, 65], 2, D, dtype, seed=29)
    inp["g"].zero_()
    out, fin = run_prefill(inp)
    check_prefill(inp, out, fin)


@pytest.mark.parametrize("D", [64, 128])
def test_degenerate_orthonormal_keys_retrieve_values_exactly(D):
    """beta = 1, alpha = 1, orthonormal keys (T <= dk), zero initial state, fp32: after
    every token t the state returns each value written so far exactly, S_t^T k_i = v_i, so
    with q_t = k_t the output is v_t; checked on the GPU's outputs and final state."""
    T, H = 48, 2
    gen = torch.Generator().manual_seed(37)
    k = torch.empty(T, H, D)
    for h in range(H):
        Q, _ = torch.linalg.qr(torch.randn(D, D, generator=gen, dtype=torch.float64))
        k[:, h] = Q[:, :T].T.float()
    inp = dict(q=k.clone(), k=k, v=torch.randn(T, H, D, generator=gen), g=torch.zeros(T, H, D),
               beta=torch.ones(T, H), cu_seqlens=torch.tensor([0, T], dtype=torch.int32), s0=None)
    out, fin = run_prefill(inp)
    v = inp["v"].double().numpy()
    kk = k.double().numpy()
    retrieved = np.einsum("hcv,thc->thv", fin[0], kk)        # S_T^T k_i for every key
    assert np.abs(retrieved - v).max() <= 1e-4 * np.abs(v).max()
    assert np.abs(out - v).max() <= 1e-4 * np.abs(v).max()


@pytest.mark.parametrize("D", [128, 64])
def test_many_one_and_two_token_sequences(D):
    """Appends of one or two tokens (a prefill of a prompt's last tokens onto a cached
    state): 400 short sequences x 4 heads, so that some q . k cancel to a small value; the
    output of a one-token slice rests on that diagonal entry, which the preparation takes in
    fp32 from the inputs.  Every slice must still meet the tolerance."""
    lens = [1 + (i % 2) for i in range(400)]
    inp = synthetic.make_prefill_inputs(lens, 4, D, D, torch.bfloat16, 3.0, 0.02, 41 + D)
    out, fin = run_prefill(inp, C=64)
    e_o, e_f = check_prefill(inp, out, fin)
    print("short sequences D=%d: max rel err out %.3g final %.3g" % (D, e_o, e_f))


def test_bf16_d64():
    inp = _inputs([130, 64, 7], 2, 64, torch.bfloat16, seed=12)
    out, fin = run_prefill(inp, C=64)
    check_prefill(inp, out, fin)


def test_bf16_d64_tensor_core_path_windows_emission_strong_decay():
    """bf16 at d = 64 runs on the tensor-core kernels as the first 64 channels of a
    128-channel problem: against the oracle per slice and per chunk, with mild and strong
    decay (g = logsigmoid(N(3, 1)) and logsigmoid(N(-3, 1))); in windows of chunks and with
    state emission, bit for bit the same as in one window."""
    lens, H = [700, 0, 333, 64, 1300], 3
    for g_mean, seed in ((3.0, 31), (-3.0, 32)):
        inp = synthetic.make_prefill_inputs(lens, H, 64, 64, torch.bfloat16, g_mean, 0.02, seed)
        out, fin = run_prefill(inp, C=64, in_flags=kda.KDA_IN_SERIAL_CHAINS)
        check_prefill(inp, out, fin, chunk=64)
        T, N = sum(lens), len(lens)
        least = kda.kda_prefill_workspace_size_min(T, N, H, 64, 64, 64, torch.bfloat16)
        ws = torch.empty(least + 4 * H * (90624 + 8) + 2048, dtype=torch.uint8, device="cuda")
        assert kda.kda_prefill_windows(T, N, H, 64, 64, 64, torch.bfloat16, ws.numel()) > 2
        d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
        pos = torch.tensor([64, 700, 700 + 320, 1097, 1097 + 1280], dtype=torch.int64, device="cuda")
        res = []
        for workspace in (None, ws):
            o = torch.full((T, H, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
            f = torch.full((N, H, 64, 64), float("nan"), device="cuda")
            e = torch.full((pos.shape[0], H, 64, 64), float("nan"), device="cuda")
            kda.kda_prefill_emit(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], o, pos, e,
                                 initial_state=d["s0"], final_state=f, workspace=workspace)
            assert kda.kda_get_device_status() == kda.KDA_OK
            res.append([x.double().cpu().numpy() for x in (o, f, e)])
        for a, b in zip(*res):
            np.testing.assert_array_equal(b, a)
        np.testing.assert_array_equal(res[0][0], out)
        # the state after 700 tokens of sequence 0 is its final state
        np.testing.assert_array_equal(res[0][2][1], res[0][1][0])


def test_config1_full_size_sampled_heads():
    """Config 1 at full size (H=32, T=8192, D=128, bf16) in the benchmark's launch
    configuration; the oracle checks every output and the final state of 3 heads."""
    inp = synthetic.make_config_inputs(1)
    out, fin = run_prefill(inp, C=64)
    e_o, e_f = check_prefill(inp, out, fin, heads=[0, 13, 31], chunk=64)
    print("config1 max rel err out %.3g final %.3g" % (e_o, e_f))


def test_config2_full_size_sampled_heads():
    """Config 2 at full size (16 sequences, lengths U[1024, 32768], S0 ~ N(0, 0.02^2))."""
    inp = synthetic.make_config_inputs(2)
    out, fin = run_prefill(inp, C=64)
    e_o, e_f = check_prefill(inp, out, fin, heads=[5, 30], chunk=64)
    print("config2 max rel err out %.3g final %.3g" % (e_o, e_f))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_continuation_equals_single_run(dtype):
    """prefill(0:T1) then prefill(T1:T, initial=final) == prefill(0:T) (append-prefill)."""
    T, T1 = 777, 300
    inp = _inputs([T], 2, 128, dtype, seed=21)
    out, fin = run_prefill(inp)
    a = {k: (v[:T1] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    a["cu_seqlens"] = torch.tensor([0, T1], dtype=torch.int32)
    oA, fA = run_prefill(a)
    b = {k: (v[T1:] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    b["cu_seqlens"] = torch.tensor([0, T - T1], dtype=torch.int32)
    b["s0"] = torch.from_numpy(fA).float()
    oB, fB = run_prefill(b)
    tol = TOL[dtype]
    import oracle
    assert oracle.rel_frobenius(np.concatenate([oA, oB]), out) <= tol
    assert oracle.rel_frobenius(fB, fin) <= tol


def test_varlen_equals_separate_runs_bitwise():
    lens = [200, 64, 1, 129]
    inp = _inputs(lens, 2, 128, torch.bfloat16, seed=31)
    out, fin = run_prefill(inp)
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        sub = {k: (v[a:b] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
        sub["cu_seqlens"] = torch.tensor([0, b - a], dtype=torch.int32)
        sub["s0"] = inp["s0"][n:n + 1]
        o_n, f_n = run_prefill(sub)
        np.testing.assert_array_equal(o_n, out[a:b])
        np.testing.assert_array_equal(f_n, fin[n:n + 1])


def test_final_state_may_alias_initial_state_and_be_null():
    inp = _inputs([100, 70], 2, 64, torch.float32, seed=41)
    out, fin = run_prefill(inp)
    d = to_device(inp)
    S = d["s0"].clone()
    out2 = torch.empty_like(d["v"])
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out2,
                    initial_state=S, final_state=S, C=64)
    np.testing.assert_array_equal(S.double().cpu().numpy(), fin)
    np.testing.assert_array_equal(out2.double().cpu().numpy(), out)
    o3, f3 = run_prefill(inp, want_final=False)
    np.testing.assert_array_equal(o3, out)


def test_zero_tokens_copies_initial_state():
    inp = _inputs([0, 0], 2, 128, torch.float32, seed=51)
    d = to_device(inp)
    sf = torch.full_like(d["s0"], float("nan"))
    out = torch.empty(0, 2, 128, device="cuda")
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                    initial_state=d["s0"], final_state=sf, C=64)
    assert kda.kda_get_device_status() == kda.KDA_OK
    assert torch.equal(sf, d["s0"])
    sf2 = torch.full_like(d["s0"], float("nan"))
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                    initial_state=None, final_state=sf2, C=64)
    assert torch.count_nonzero(sf2) == 0


def test_bad_cu_seqlens_reported_by_device():
    """cu_seqlens that do not end at total_tokens (or decrease) are detected on the
    device and reported through the status word; no out-of-range access happens
    because each CTA validates its own sequence bounds before touching tokens."""
    inp = _inputs([40, 40], 2, 64, torch.float32, seed=61)
    d = to_device(inp)
    out = torch.empty_like(d["v"])
    bad = torch.tensor([0, 50, 30], dtype=torch.int32, device="cuda")   # decreasing, short
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], bad, out, C=64)
    assert kda.kda_get_device_status() == kda.KDA_ERR_BAD_SEQLENS
    assert kda.kda_get_device_status() == kda.KDA_OK   # cleared by the read


@pytest.mark.slow
def test_config4_long_context_full_size_sampled_heads():
    """Config 4 at full size: T = 1,048,576, H = 32, D = 128, bf16, slow decay
    g = logsigmoid(N(4, 1)), zero initial state, in the benchmark's launch configuration.
    Heads 0 and 17 are drawn on the CPU and followed by the fp64 oracle over all 1M tokens
    (every output row and the final state); the other heads are drawn on the device."""
    import oracle
    cfg = synthetic.CONFIGS[4]
    lens = synthetic.draw_lengths(cfg)
    heads = [0, 17]
    d = synthetic.make_prefill_inputs_device(lens, cfg.H, cfg.D, cfg.D, cfg.dtype, cfg.g_mean,
                                             cfg.s0_std, cfg.seed, cpu_heads=heads)
    T = sum(lens)
    out = torch.empty(T, cfg.H, cfg.D, dtype=cfg.dtype, device="cuda")
    fin = torch.empty(1, cfg.H, cfg.D, cfg.D, device="cuda")
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                    final_state=fin, C=cfg.C)
    assert kda.kda_get_device_status() == kda.KDA_OK
    o = out[:, heads].double().cpu().numpy()
    f = fin[:, heads].double().cpu().numpy()
    del d["q"], d["k"], d["v"], d["g"], out
    c = d["cpu"]
    o_ref, f_ref = oracle.prefill(c["q"], c["k"], c["v"], c["g"], c["beta"], c["cu_seqlens"],
                                  nthreads=len(heads))
    e_o = oracle.max_rel_frobenius_per_slice(o, o_ref, c["cu_seqlens"])
    e_f = oracle.max_rel_frobenius_states(f, f_ref)
    e_c = oracle.max_rel_frobenius_per_chunk(o, o_ref, c["cu_seqlens"], cfg.C)
    print("config4 max rel err out %.3g final %.3g worst chunk %.3g" % (e_o, e_f, e_c))
    assert e_o <= TOL[torch.bfloat16] and e_f <= TOL[torch.bfloat16]
    assert e_c <= TOL[torch.bfloat16]
    # windows along the sequence (early, middle, end) stay within tolerance too
    for a in (0, T // 2, T - 65536):
        e_w = oracle.rel_frobenius(o[a:a + 65536], o_ref[a:a + 65536])
        assert e_w <= TOL[torch.bfloat16], (a, e_w)


@pytest.mark.parametrize("lens,H,D,windows", [
    ([8192], 32, 128, False),
    ([2048, 700, 0, 3333, 64], 32, 128, False),
    ([2048, 700, 0, 3333, 64], 32, 128, True),    # a workspace of a few windows
    ([2048, 700, 0, 3333, 64], 32, 64, False),    # d = 64 on the tensor cores
    ([262144], 4, 128, False),                     # few long chains: the chunk-parallel scan
])
def test_bf16_prefill_is_deterministic(lens, H, D, windows):
    """Repeated calls on the same inputs give the same bits.  The tensor-core kernels pass
    data between warps through named barriers and between products through Tensor Memory;
    a missing ordering there shows up as run-to-run differences far below the parity
    tolerance, which only this comparison sees."""
    d = to_device(_inputs(lens, H, D, torch.bfloat16, seed=23))
    T, N = sum(lens), len(lens)
    if H == 4:
        assert kda.kda_prefill_launches(T, N, H, D, D, 64, torch.bfloat16) == 7   # the scan runs
    size = kda.kda_prefill_workspace_size(T, N, H, D, D, 64, torch.bfloat16)
    if windows:
        size = kda.kda_prefill_workspace_size_min(T, N, H, D, D, 64, torch.bfloat16) + 4 * H * (90624 + 8) + 2048
        assert kda.kda_prefill_windows(T, N, H, D, D, 64, torch.bfloat16, size) > 1
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    runs = []
    for _ in range(3):
        out = torch.full((T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        fin = torch.full((N, H, D, D), float("nan"), device="cuda")
        kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out,
                        initial_state=d["s0"], final_state=fin, workspace=ws)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == kda.KDA_OK
        runs.append((out.view(torch.int16).cpu().numpy(), fin.view(torch.int32).cpu().numpy()))
    for o, f in runs[1:]:
        np.testing.assert_array_equal(o, runs[0][0])
        np.testing.assert_array_equal(f, runs[0][1])
