"""Thin Python binding of libkda (ctypes).  Argument marshalling only.

Every function has the name of the C entry point it calls (include/libkda.h) and
passes torch tensors' device pointers, sizes and the current CUDA stream straight
through; all of the computation runs in the library's kernels.  There is no
fallback: if libkda.so is missing or a call fails, a RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_CUDA = 3
KDA_ERR_TIMEOUT = 4
KDA_ERR_BAD_SEQLENS = 5
KDA_ERR_BAD_EMIT_POS = 6
# input prologue flags (kda_prefill_ex / kda_decode_ex)
KDA_IN_NORMALIZE_QK = 1
KDA_IN_G_LOGITS = 2
KDA_IN_BETA_LOGITS = 4
KDA_IN_G_SCALAR = 8
KDA_IN_STRONG_DECAY = 16
KDA_IN_SERIAL_CHAINS = 32
KDA_F32 = 0
KDA_BF16 = 1

# Every symbol include/libkda.h declares (checked by the CPU tests).
EXPORTED = ("kda_prefill", "kda_prefill_workspace_size", "kda_decode", "kda_status_string",
            "kda_get_device_status", "kda_abi_version", "kda_prefill_noalloc",
            "kda_prefill_prepare", "kda_prefill_scan", "kda_selftest_bounded_wait",
            "kda_prefill_emit", "kda_prefill_gdn", "kda_decode_gdn", "kda_prefill_ex",
            "kda_decode_ex", "kda_prefill_launches", "kda_prefill_workspace_size_min",
            "kda_prefill_windows")

# Size of the library-owned scratch behind kda_prefill_noalloc (KDA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__("%s failed: %s (status %d)" % (fn, kda_status_string(status), status))
        self.status = status


def load() -> ctypes.CDLL:
    """Load libkda.so (built in-tree by linear_attention_rule_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libkda.so is not built (%s); run __graft_entry__.build()" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.kda_prefill.argtypes = [P, P, P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int, P, P,
                                I32, P, SZ, P]
    lib.kda_prefill.restype = ctypes.c_int
    lib.kda_prefill_workspace_size.argtypes = [I64, I32, I32, I32, I32, I32, ctypes.c_int]
    lib.kda_prefill_workspace_size.restype = SZ
    lib.kda_prefill_workspace_size_min.argtypes = [I64, I32, I32, I32, I32, I32, ctypes.c_int]
    lib.kda_prefill_workspace_size_min.restype = SZ
    lib.kda_prefill_windows.argtypes = [I64, I32, I32, I32, I32, I32, ctypes.c_int, SZ]
    lib.kda_prefill_windows.restype = I64
    lib.kda_decode.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, ctypes.c_int, P]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_get_device_status.argtypes = [P]
    lib.kda_get_device_status.restype = ctypes.c_int
    lib.kda_abi_version.argtypes = []
    lib.kda_abi_version.restype = I32
    lib.kda_prefill_noalloc.argtypes = [P, P, P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int,
                                        P, P, I32, P]
    lib.kda_prefill_noalloc.restype = ctypes.c_int
    lib.kda_prefill_prepare.argtypes = [P, P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int, I32,
                                        P, SZ, P]
    lib.kda_prefill_prepare.restype = ctypes.c_int
    lib.kda_prefill_scan.argtypes = [P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int, I32, P, SZ, P]
    lib.kda_prefill_scan.restype = ctypes.c_int
    U32 = ctypes.c_uint32
    lib.kda_prefill_ex.argtypes = [P, P, P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int, P, P,
                                   I32, U32, P, I32, P, P, SZ, P]
    lib.kda_prefill_ex.restype = ctypes.c_int
    lib.kda_decode_ex.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, ctypes.c_int, U32, P]
    lib.kda_decode_ex.restype = ctypes.c_int
    lib.kda_prefill_gdn.argtypes = list(lib.kda_prefill.argtypes)
    lib.kda_prefill_gdn.restype = ctypes.c_int
    lib.kda_decode_gdn.argtypes = list(lib.kda_decode.argtypes)
    lib.kda_decode_gdn.restype = ctypes.c_int
    lib.kda_prefill_emit.argtypes = [P, P, P, P, P, P, P, I32, I64, I32, I32, I32, ctypes.c_int, P, P,
                                     I32, P, I32, P, P, SZ, P]
    lib.kda_prefill_emit.restype = ctypes.c_int
    lib.kda_prefill_launches.argtypes = [I64, I32, I32, I32, I32, I32, ctypes.c_int, U32, I32]
    lib.kda_prefill_launches.restype = I32
    lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_uint64, P]
    lib.kda_selftest_bounded_wait.restype = ctypes.c_int
    _lib = lib
    return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError("q/k/v/out must be float32 or bfloat16, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libkda must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check(device, **args):
    """Validate the tensors of one call before any pointer reaches the library: each value
    is (tensor or None, expected shape, expected dtype).  Shapes and dtypes are checked
    first, then that every tensor is contiguous and on `device` (the device of q or out),
    so a mistake raises here instead of becoming an out-of-bounds access on the GPU."""
    for name, (t, shape, dtype) in args.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError("%s must be a torch.Tensor" % name)
        if t.dtype != dtype:
            raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
        if tuple(t.shape) != tuple(shape):
            raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    for name, (t, _, _) in args.items():
        if t is None:
            continue
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
        if t.device.type != "cuda" or t.device != device:
            raise ValueError("%s must be on %s (libkda takes device pointers), got %s"
                             % (name, device, t.device))


def _check_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state, final_state, scalar_g=False,
                   workspace=None, emit_pos=None, emit_states=None):
    """Shapes of a prefill call: q, k [T, H, dk], v, out [T, H, dv] in q's dtype; g [T, H, dk]
    (or [T, H] for a scalar gate) and beta [T, H] fp32; cu_seqlens int32 [N+1]; states fp32
    [N, H, dk, dv]; workspace uint8 (its size is checked by the library); emission positions
    int64 [E] with their states fp32 [E, H, dk, dv]."""
    if q.dim() != 3 or v.dim() != 3 or cu_seqlens.dim() != 1:
        raise ValueError("q and v must be [T, H, d] and cu_seqlens [N+1]")
    if (emit_pos is None) != (emit_states is None):
        raise ValueError("emit_pos and emit_states go together")
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    E = emit_pos.shape[0] if emit_pos is not None and emit_pos.dim() == 1 else -1
    dt = q.dtype
    _check(q.device, q=(q, (T, H, dk), dt), k=(k, (T, H, dk), dt), v=(v, (T, H, dv), dt),
           out=(out, (T, H, dv), dt), g=(g, (T, H) if scalar_g else (T, H, dk), torch.float32),
           beta=(beta, (T, H), torch.float32), cu_seqlens=(cu_seqlens, (N + 1,), torch.int32),
           initial_state=(initial_state, (N, H, dk, dv), torch.float32),
           final_state=(final_state, (N, H, dk, dv), torch.float32),
           workspace=(workspace, (workspace.numel(),) if workspace is not None else (), torch.uint8),
           emit_pos=(emit_pos, (E,), torch.int64),
           emit_states=(emit_states, (E, H, dk, dv), torch.float32))


def _check_decode(q, k, v, g, beta, state, out, scalar_g=False):
    """Shapes of a decode call: q, k [N, H, dk], v, out [N, H, dv] in q's dtype; g [N, H, dk]
    (or [N, H]) and beta [N, H] fp32; state fp32 [N, H, dk, dv]."""
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q and v must be [N, H, d]")
    N, H, dk = q.shape
    dv = v.shape[2]
    dt = q.dtype
    _check(q.device, q=(q, (N, H, dk), dt), k=(k, (N, H, dk), dt), v=(v, (N, H, dv), dt),
           out=(out, (N, H, dv), dt), g=(g, (N, H) if scalar_g else (N, H, dk), torch.float32),
           beta=(beta, (N, H), torch.float32), state=(state, (N, H, dk, dv), torch.float32))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def kda_status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def kda_abi_version() -> int:
    return int(load().kda_abi_version())


def kda_prefill_workspace_size(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int,
                               C: int, dtype: torch.dtype) -> int:
    code = KDA_F32 if dtype == torch.float32 else KDA_BF16
    return int(load().kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv, C, code))


def kda_prefill_workspace_size_min(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int,
                                   C: int, dtype: torch.dtype) -> int:
    """The least workspace the prefill accepts; below kda_prefill_workspace_size it runs the
    chunks in windows (kda_prefill_workspace_size_min in include/libkda.h)."""
    code = KDA_F32 if dtype == torch.float32 else KDA_BF16
    return int(load().kda_prefill_workspace_size_min(total_tokens, num_seqs, H, dk, dv, C, code))


def kda_prefill_windows(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int, C: int,
                        dtype: torch.dtype, ws_bytes: int) -> int:
    """Windows a prefill with a workspace of ws_bytes runs in (kda_prefill_windows in
    include/libkda.h); -1 when the workspace is too small or the problem unsupported."""
    code = KDA_F32 if dtype == torch.float32 else KDA_BF16
    return int(load().kda_prefill_windows(total_tokens, num_seqs, H, dk, dv, C, code, ws_bytes))


def kda_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state=None, final_state=None,
                C: int = 64, workspace: Optional[torch.Tensor] = None, stream=None):
    """Chunkwise KDA prefill (see kda_prefill in include/libkda.h).

    q, k [T, H, dk], v/out [T, H, dv] (fp32 or bf16); g [T, H, dk] and beta [T, H] fp32;
    cu_seqlens int32 [N+1] on the device; initial_state / final_state fp32 [N, H, dk, dv]
    or None.  The workspace is allocated with torch when not given.
    """
    return _prefill("kda_prefill", q, k, v, g, beta, cu_seqlens, out, initial_state, final_state,
                    C, workspace, stream)


def kda_prefill_gdn(q, k, v, g, beta, cu_seqlens, out, initial_state=None, final_state=None,
                    C: int = 64, workspace: Optional[torch.Tensor] = None, stream=None):
    """Gated DeltaNet prefill: kda_prefill with a scalar gate g [T, H] fp32 (kda_prefill_gdn
    in include/libkda.h)."""
    return _prefill("kda_prefill_gdn", q, k, v, g, beta, cu_seqlens, out, initial_state,
                    final_state, C, workspace, stream)


def _prefill(fn, q, k, v, g, beta, cu_seqlens, out, initial_state, final_state, C, workspace, stream):
    lib = load()
    dt = _dtype_code(q)
    _check_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state, final_state,
                   scalar_g=fn == "kda_prefill_gdn", workspace=workspace)
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    need = int(lib.kda_prefill_workspace_size(T, N, H, dk, dv, C, dt))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                          _ptr(cu_seqlens), N, T, H, dk, dv, dt, _ptr(out), _ptr(final_state), C,
                          _ptr(workspace), ws_bytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError(fn, st)
    return out, final_state


def kda_prefill_emit(q, k, v, g, beta, cu_seqlens, out, emit_pos, emit_states,
                     initial_state=None, final_state=None, C: int = 64,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """kda_prefill that also writes the state at the token boundaries emit_pos (int64 [E],
    device) into emit_states (fp32 [E, H, dk, dv]); see kda_prefill_emit in
    include/libkda.h."""
    lib = load()
    dt = _dtype_code(q)
    _check_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state, final_state, workspace=workspace,
                   emit_pos=emit_pos, emit_states=emit_states)
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    need = int(lib.kda_prefill_workspace_size(T, N, H, dk, dv, C, dt))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.kda_prefill_emit(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                              _ptr(cu_seqlens), N, T, H, dk, dv, dt, _ptr(out), _ptr(final_state), C,
                              _ptr(emit_pos), int(emit_pos.shape[0]), _ptr(emit_states),
                              _ptr(workspace), ws_bytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_prefill_emit", st)
    return out, final_state, emit_states


def kda_prefill_ex(q, k, v, g, beta, cu_seqlens, out, in_flags: int = 0, initial_state=None,
                   final_state=None, emit_pos=None, emit_states=None, C: int = 64,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """kda_prefill with an input prologue (KDA_IN_* flags) and optional state emission
    (kda_prefill_ex in include/libkda.h).  With KDA_IN_G_SCALAR, g is [T, H]."""
    lib = load()
    dt = _dtype_code(q)
    _check_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state, final_state,
                   scalar_g=bool(int(in_flags) & KDA_IN_G_SCALAR), workspace=workspace,
                   emit_pos=emit_pos, emit_states=emit_states)
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    need = int(lib.kda_prefill_workspace_size(T, N, H, dk, dv, C, dt))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    num_emit = 0 if emit_pos is None else int(emit_pos.shape[0])
    st = lib.kda_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                            _ptr(cu_seqlens), N, T, H, dk, dv, dt, _ptr(out), _ptr(final_state), C,
                            int(in_flags), _ptr(emit_pos), num_emit, _ptr(emit_states),
                            _ptr(workspace), ws_bytes, _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_prefill_ex", st)
    return out, final_state


def kda_prefill_noalloc(q, k, v, g, beta, cu_seqlens, out, initial_state=None,
                        final_state=None, C: int = 64, stream=None):
    """kda_prefill without a workspace, for callers that cannot allocate device memory
    where they run (their memory belongs to another allocator, or an allocation's stall
    is not acceptable): the library's own static scratch is used instead.  bf16 with
    d = 128 and C = 64 only; problems needing more than NOALLOC_SCRATCH_BYTES of scratch
    are rejected.  Calls sharing a device must not overlap on the GPU."""
    lib = load()
    _dtype_code(q)
    _check_prefill(q, k, v, g, beta, cu_seqlens, out, initial_state, final_state)
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    st = lib.kda_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(initial_state), _ptr(cu_seqlens), N, T, H, dk, dv,
                                 _dtype_code(q), _ptr(out), _ptr(final_state), C, _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_prefill_noalloc", st)
    return out, final_state


def _ws(workspace):
    return 0 if workspace is None else workspace.numel() * workspace.element_size()


def kda_prefill_prepare(q, k, v, g, beta, cu_seqlens, workspace, C: int = 64, stream=None):
    """Stage 1 of the tensor-core prefill (chunk table + preparation) into `workspace`."""
    lib = load()
    _dtype_code(q)
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q and v must be [T, H, d]")
    _check_prefill(q, k, v, g, beta, cu_seqlens, None, None, None, workspace=workspace)
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    st = lib.kda_prefill_prepare(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N,
                                 T, H, dk, dv, _dtype_code(q), C, _ptr(workspace), _ws(workspace),
                                 _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_prefill_prepare", st)


def kda_prefill_scan(out, cu_seqlens, workspace, initial_state=None, final_state=None,
                     C: int = 64, stream=None):
    """Stage 2: the chunk recurrence with the chunk outputs beside it; reads initial_state,
    writes `out` [T, H, D] bf16 and final_state."""
    lib = load()
    _dtype_code(out)
    if out.dim() != 3 or cu_seqlens.dim() != 1:
        raise ValueError("out must be [T, H, D] and cu_seqlens [N+1]")
    T, H, D = out.shape
    N = cu_seqlens.shape[0] - 1
    _check(out.device, out=(out, (T, H, D), out.dtype), cu_seqlens=(cu_seqlens, (N + 1,), torch.int32),
           initial_state=(initial_state, (N, H, D, D), torch.float32),
           final_state=(final_state, (N, H, D, D), torch.float32),
           workspace=(workspace, (workspace.numel(),) if workspace is not None else (), torch.uint8))
    st = lib.kda_prefill_scan(_ptr(initial_state), _ptr(final_state), _ptr(out), _ptr(cu_seqlens), N,
                              T, H, D, D, _dtype_code(out), C, _ptr(workspace), _ws(workspace),
                              _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_prefill_scan", st)


def kda_selftest_bounded_wait(limit_ns: int, stream=None):
    """Launch the bounded-wait self-test; read the outcome with kda_get_device_status."""
    st = load().kda_selftest_bounded_wait(int(limit_ns), _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_selftest_bounded_wait", st)


def kda_decode(q, k, v, g, beta, state, out, stream=None):
    """One KDA decode step in place on `state` [N, H, dk, dv] fp32 (kda_decode in libkda.h)."""
    return _decode("kda_decode", q, k, v, g, beta, state, out, stream)


def kda_decode_gdn(q, k, v, g, beta, state, out, stream=None):
    """One Gated DeltaNet decode step: kda_decode with a scalar gate g [N, H] fp32."""
    return _decode("kda_decode_gdn", q, k, v, g, beta, state, out, stream)


def kda_decode_ex(q, k, v, g, beta, state, out, in_flags: int = 0, stream=None):
    """kda_decode with an input prologue (KDA_IN_* flags; with KDA_IN_G_SCALAR g is [N, H])."""
    lib = load()
    _dtype_code(q)
    _check_decode(q, k, v, g, beta, state, out, scalar_g=bool(int(in_flags) & KDA_IN_G_SCALAR))
    N, H, dk = q.shape
    dv = v.shape[2]
    st = lib.kda_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                           N, H, dk, dv, _dtype_code(q), int(in_flags), _stream(stream))
    if st != KDA_OK:
        raise KdaError("kda_decode_ex", st)
    return out


def _decode(fn, q, k, v, g, beta, state, out, stream):
    lib = load()
    _dtype_code(q)
    _check_decode(q, k, v, g, beta, state, out, scalar_g=fn == "kda_decode_gdn")
    N, H, dk = q.shape
    dv = v.shape[2]
    st = getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                          N, H, dk, dv, _dtype_code(q), _stream(stream))
    if st != KDA_OK:
        raise KdaError(fn, st)
    return out


def kda_get_device_status(stream=None) -> int:
    """Synchronise `stream`, return and clear the device status word."""
    return int(load().kda_get_device_status(_stream(stream)))


def tensor_core_path(dtype: torch.dtype, D: int) -> bool:
    # mirrors tensor_core_path() in csrc/libkda.cu
    return dtype == torch.bfloat16 and D == 128


def kda_prefill_launches(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int, C: int,
                         dtype: torch.dtype, in_flags: int = 0, num_emit: int = 0) -> int:
    """Kernels one kda_prefill_ex call with these sizes launches (kda_prefill_launches in
    include/libkda.h)."""
    code = KDA_F32 if dtype == torch.float32 else KDA_BF16
    return int(load().kda_prefill_launches(total_tokens, num_seqs, H, dk, dv, C, code, in_flags, num_emit))


def prefill_compute_dtype(dtype: torch.dtype, D: int = 128) -> str:
    """Operand type of the prefill contractions (accumulation and the state are fp32
    on every path)."""
    return "bf16" if tensor_core_path(dtype, D) else "f32"
