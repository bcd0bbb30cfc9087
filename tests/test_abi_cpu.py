"""CPU checks of the C-ABI library: it loads, exports every symbol the header declares,
and rejects bad arguments with a status before launching anything (no GPU needed:
argument checks return before any CUDA call)."""
import ctypes
import os
import re

import pytest

from linear_attention_rule_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_rule_b200 import build
    build.build()
    return kda.load()


def declared_functions():
    with open(os.path.join(ROOT, "include", "libkda.h")) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    assert set(declared_functions()) == set(kda.EXPORTED)


def test_header_constants_match_the_binding():
    """Every KDA_* enum value the header declares has the same value in the binding."""
    with open(os.path.join(ROOT, "include", "libkda.h")) as fh:
        text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
    consts = dict((n, int(v)) for n, v in re.findall(r"\b(KDA_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert len(consts) >= 13
    for name, value in consts.items():
        assert getattr(kda, name) == value, name


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    assert kda.kda_abi_version() == 8
    for code in range(7):
        s = kda.kda_status_string(code)
        assert s and s != "unknown status"
    assert kda.kda_status_string(99) == "unknown status"


def _prefill(lib, **kw):
    P = ctypes.c_void_p
    a = dict(q=P(4096), k=P(4096), v=P(4096), g=P(4096), beta=P(4096), s0=None, cu=P(4096),
             N=1, T=64, H=2, dk=64, dv=64, dt=kda.KDA_F32, out=P(4096), sf=None, C=64,
             ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.kda_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s0"], a["cu"], a["N"],
                           a["T"], a["H"], a["dk"], a["dv"], a["dt"], a["out"], a["sf"], a["C"],
                           a["ws"], a["ws_bytes"], a["stream"])


def test_prefill_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    assert _prefill(lib, H=0) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, N=-1) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, T=-5) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, dt=7) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, dk=96, dv=96) == kda.KDA_ERR_UNSUPPORTED
    assert _prefill(lib, dk=64, dv=128) == kda.KDA_ERR_UNSUPPORTED
    assert _prefill(lib, C=48) == kda.KDA_ERR_UNSUPPORTED
    assert _prefill(lib, dt=kda.KDA_BF16, C=32) == kda.KDA_ERR_UNSUPPORTED
    assert _prefill(lib, T=1 << 31) == kda.KDA_ERR_UNSUPPORTED
    assert _prefill(lib, cu=None) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, out=None) == kda.KDA_ERR_INVALID_ARG
    assert _prefill(lib, k=P(4100)) == kda.KDA_ERR_INVALID_ARG       # misaligned
    assert _prefill(lib, sf=P(4104)) == kda.KDA_ERR_INVALID_ARG      # misaligned
    assert _prefill(lib, cu=P(4098)) == kda.KDA_ERR_INVALID_ARG      # misaligned int32
    # nothing to do: valid, returns before touching the device
    assert _prefill(lib, N=0) == kda.KDA_OK


def test_prefill_workspace_check(lib):
    need = lib.kda_prefill_workspace_size_min(8192, 1, 32, 128, 128, 64, kda.KDA_BF16)
    if need > 0:
        assert _prefill(lib, dk=128, dv=128, H=32, T=8192, dt=kda.KDA_BF16,
                        ws=ctypes.c_void_p(4096), ws_bytes=need - 1) == kda.KDA_ERR_INVALID_ARG
        assert _prefill(lib, dk=128, dv=128, H=32, T=8192, dt=kda.KDA_BF16,
                        ws=ctypes.c_void_p(4096 + 16), ws_bytes=need) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_prefill_workspace_size(100, 1, 2, 96, 96, 64, kda.KDA_F32) == 0
    assert lib.kda_prefill_workspace_size(-1, 1, 2, 64, 64, 64, kda.KDA_F32) == 0


def test_decode_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    def dec(**kw):
        a = dict(q=P(4096), k=P(4096), v=P(4096), g=P(4096), beta=P(4096), S=P(4096), out=P(4096),
                 N=4, H=2, dk=128, dv=128, dt=kda.KDA_BF16, stream=None)
        a.update(kw)
        return lib.kda_decode(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S"], a["out"], a["N"],
                              a["H"], a["dk"], a["dv"], a["dt"], a["stream"])
    assert dec(N=-1) == kda.KDA_ERR_INVALID_ARG
    assert dec(H=0) == kda.KDA_ERR_INVALID_ARG
    assert dec(dk=32, dv=32) == kda.KDA_ERR_UNSUPPORTED
    assert dec(S=None) == kda.KDA_ERR_INVALID_ARG
    assert dec(g=P(4097)) == kda.KDA_ERR_INVALID_ARG
    assert dec(dt=5) == kda.KDA_ERR_INVALID_ARG
    assert dec(N=0) == kda.KDA_OK


def test_staged_entry_points_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    need = lib.kda_prefill_workspace_size(256, 1, 2, 128, 128, 64, kda.KDA_BF16)
    ws = P(1 << 20)
    # only the tensor-core problem is staged
    assert lib.kda_prefill_prepare(P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), 1, 256, 2,
                                   64, 64, kda.KDA_F32, 64, ws, need, None) == kda.KDA_ERR_UNSUPPORTED
    out = P(8192)
    assert lib.kda_prefill_scan(None, None, out, P(4096), 1, 256, 2, 128, 128, kda.KDA_BF16, 64, ws,
                                need - 1, None) == kda.KDA_ERR_INVALID_ARG
    # out is required once there are tokens, and must be 16-byte aligned
    assert lib.kda_prefill_scan(None, None, None, P(4096), 1, 256, 2, 128, 128, kda.KDA_BF16, 64, ws,
                                need, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_prefill_scan(None, None, P(8192 + 8), P(4096), 1, 256, 2, 128, 128, kda.KDA_BF16,
                                64, ws, need, None) == kda.KDA_ERR_INVALID_ARG
    # misaligned workspace
    assert lib.kda_prefill_scan(None, None, out, P(4096), 1, 256, 2, 128, 128, kda.KDA_BF16, 64,
                                P((1 << 20) + 16), need, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_prefill_scan(None, None, None, P(4096), 0, 0, 2, 128, 128, kda.KDA_BF16, 64, ws,
                                need, None) == kda.KDA_OK


def test_emit_entry_point_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    need = lib.kda_prefill_workspace_size(256, 1, 2, 128, 128, 64, kda.KDA_BF16)
    ws = P(1 << 20)

    def emit(dt=kda.KDA_BF16, dk=128, N=1, pos=P(4096), num=2, st=P(8192)):
        return lib.kda_prefill_emit(P(4096), P(4096), P(4096), P(4096), P(4096), None, P(4096), N,
                                    256, 2, dk, dk, dt, P(4096), None, 64, pos, num, st, ws, need, None)
    assert emit(num=-1) == kda.KDA_ERR_INVALID_ARG
    assert emit(pos=None) == kda.KDA_ERR_INVALID_ARG
    assert emit(st=None) == kda.KDA_ERR_INVALID_ARG
    assert emit(pos=P(4100)) == kda.KDA_ERR_INVALID_ARG       # emit_pos must be 8-byte aligned
    assert emit(st=P(8200)) == kda.KDA_ERR_INVALID_ARG        # emit_states 16-byte aligned
    assert emit(N=0) == kda.KDA_ERR_INVALID_ARG               # positions but no sequence
    assert emit(dt=kda.KDA_F32) == kda.KDA_ERR_UNSUPPORTED    # emission: tensor-core path only
    assert emit(dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert kda.kda_status_string(kda.KDA_ERR_BAD_EMIT_POS) != "unknown status"


def test_gdn_entry_points_check_arguments_like_kda(lib):
    P = ctypes.c_void_p
    assert lib.kda_prefill_gdn(P(4096), P(4096), P(4096), P(4096), P(4096), None, P(4096), 1, 256, 2,
                               32, 32, kda.KDA_BF16, P(4096), None, 64, None, 0, None) == kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_prefill_gdn(P(4096), P(4096), P(4096), P(4100), P(4096), None, P(4096), 1, 256, 2,
                               64, 64, kda.KDA_F32, P(4096), None, 64, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_gdn(P(4096), P(4096), P(4096), None, P(4096), P(4096), P(4096), 4, 2, 128, 128,
                              kda.KDA_BF16, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_gdn(P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), 0, 2, 128,
                              128, kda.KDA_BF16, None) == kda.KDA_OK


def test_prologue_entry_points_reject_unknown_flags(lib):
    P = ctypes.c_void_p
    need = lib.kda_prefill_workspace_size(256, 1, 2, 128, 128, 64, kda.KDA_BF16)
    ex = lambda flags: lib.kda_prefill_ex(P(4096), P(4096), P(4096), P(4096), P(4096), None, P(4096), 1, 256,
                                          2, 128, 128, kda.KDA_BF16, P(4096), None, 64, flags, None, 0, None,
                                          P(1 << 20), need, None)
    assert ex(64) == kda.KDA_ERR_INVALID_ARG
    assert ex(1 << 31) == kda.KDA_ERR_INVALID_ARG
    dec = lambda flags: lib.kda_decode_ex(P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), 2,
                                          2, 128, 128, kda.KDA_BF16, flags, None)
    assert dec(64) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_ex(P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), P(4096), 0, 2, 128, 128,
                             kda.KDA_BF16, 63, None) == kda.KDA_OK   # every known bit, N = 0


def test_selftest_rejects_out_of_range_limits(lib):
    assert lib.kda_selftest_bounded_wait(10, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_selftest_bounded_wait(3_000_000_000, None) == kda.KDA_ERR_INVALID_ARG


def test_prefill_launch_count(lib):
    """Host-side count of the kernels one prefill call launches (no device needed)."""
    bf, f32 = kda.KDA_BF16, kda.KDA_F32
    n = lambda T, N, H, dt=bf, flags=0, emit=0, d=128: lib.kda_prefill_launches(T, N, H, d, d, 64, dt, flags, emit)
    assert n(8192, 1, 32) == 4                    # 128 chunks per chain: segments too short
    assert n(1 << 20, 1, 32) == 4                 # 32 chains x 4 slices already fill the SMs
    assert n(1 << 20, 1, 8) == 7                  # 8 long chains: chunk-parallel scan (+3)
    assert n(1 << 20, 1, 8, flags=kda.KDA_IN_SERIAL_CHAINS) == 4
    assert n(8192, 16, 32) == 5                   # 512 chains fill the SMs: no scan; +1: the sequences' order
    assert n(300, 1, 2) == 4                      # 5 chunks per chain: segments too short
    assert n(8192, 1, 32, emit=2) == 5
    assert n(0, 1, 32) == 2                       # chunk table and recurrence only
    assert n(8192, 0, 32) == 0
    assert n(256, 1, 2, dt=f32, d=64) == 1        # CUDA-core path: one kernel
    assert n(256, 1, 2, d=64) == 4                # bf16 at d = 64: the tensor-core kernels
    assert n(1 << 20, 1, 8, d=64) == 7            # the chunk-parallel scan at d = 64 too
    assert n(256, 1, 2, d=96) == -1


REC = 90624   # bytes of one chunk record (one chunk of 64 tokens, one head)


def test_window_workspace_sizes(lib):
    """Below the full workspace the prefill runs in windows of W chunks: the least
    workspace is windows of 8 chunks, and the count of windows follows from the bytes."""
    bf = kda.KDA_BF16
    full = lambda T, N, H: lib.kda_prefill_workspace_size(T, N, H, 128, 128, 64, bf)
    least = lambda T, N, H: lib.kda_prefill_workspace_size_min(T, N, H, 128, 128, 64, bf)
    win = lambda T, N, H, ws: lib.kda_prefill_windows(T, N, H, 128, 128, 64, bf, ws)
    T, N, H = 8192, 1, 32
    mc = T // 64 + N                                   # chunks the layout reserves
    assert win(T, N, H, full(T, N, H)) == 1
    lo = least(T, N, H)
    # 8 chunks of records, two carried states per head, and per-chunk tables (16 B each)
    records, carry = 8 * H * REC, 2 * H * 128 * 128 * 4
    assert records + carry < lo < records + carry + 16 * mc + 64 * 1024
    assert win(T, N, H, lo) == -(-mc // 8)
    assert win(T, N, H, lo - 1) == -1
    prev = None
    for ws in (lo, lo + 5 * H * REC, lo + 40 * H * REC, full(T, N, H) - 1, full(T, N, H)):
        n = win(T, N, H, ws)
        assert n >= 1 and (prev is None or n <= prev)
        prev = n
    assert win(T, N, H, full(T, N, H) - 1) >= 2
    # a problem of at most 8 chunks needs its full workspace
    assert least(300, 1, 2) == full(300, 1, 2) and win(300, 1, 2, full(300, 1, 2)) == 1
    # the full size grows with T, the least almost not (16 bytes per chunk)
    assert full(1 << 20, 1, 32) > 40 * 10**9
    assert least(1 << 20, 1, 32) - least(8192, 1, 32) == 16 * ((1 << 20) // 64 - 8192 // 64)
    # paths that need no workspace
    assert lib.kda_prefill_workspace_size_min(256, 1, 2, 64, 64, 64, kda.KDA_F32) == 0
    assert lib.kda_prefill_windows(256, 1, 2, 64, 64, 64, kda.KDA_F32, 0) == 1
    assert lib.kda_prefill_windows(256, 1, 2, 96, 96, 64, bf, 1 << 30) == -1
