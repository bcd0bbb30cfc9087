"""White-box check of the preparation kernels: decode the per-(chunk, head) workspace record
(shared-memory operand images with a 128- or 64-byte swizzle: [M ; P] K-major, K_res,
Aqk K-major, U, gamma) and compare every chunk tensor with the fp64 chunked
form of the oracle: P = Q_dec - Aqk W, M = -K_res^T W, K_res, U, Aqk, gamma.  The recurrence adds K_res^T U and Aqk U to its products, so the
derived B = K_res^T U and R = Aqk U are checked too."""
import numpy as np
import pytest
import torch

from oracle import chunked
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import to_device

pytestmark = pytest.mark.gpu

REC_BYTES = 90624


def _bf16(u8: np.ndarray) -> np.ndarray:
    u16 = u8.copy().view(np.uint16).astype(np.uint32) << 16
    return u16.view(np.float32).astype(np.float64)


def _sw128(img: np.ndarray, rows: int) -> np.ndarray:
    """bf16 image of `rows` rows x 64 elements, 128-byte swizzle -> float array."""
    b = img[: rows * 128].reshape(rows, 8, 16)
    out = np.empty_like(b)
    for r in range(rows):
        for ch in range(8):
            out[r, ch] = b[r, ch ^ (r % 8)]
    return _bf16(out.reshape(rows, 128))


def _sw64(img: np.ndarray, rows: int) -> np.ndarray:
    """bf16 image of `rows` rows x 32 elements, 64-byte swizzle -> float array."""
    b = img[: rows * 64].reshape(rows, 4, 16)
    out = np.empty_like(b)
    for r in range(rows):
        for ch in range(4):
            out[r, ch] = b[r, ch ^ ((r // 2) % 4)]
    return _bf16(out.reshape(rows, 64))


def _records(nrow, seed, g_mean):
    inp = synthetic.make_prefill_inputs([nrow], 1, 128, 128, torch.bfloat16, g_mean, 0.0, seed)
    d = to_device(inp)
    need = kda.kda_prefill_workspace_size(nrow, 1, 1, 128, 128, 64, torch.bfloat16)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    kda.kda_prefill_prepare(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], ws, C=64)
    assert kda.kda_get_device_status() == kda.KDA_OK
    return inp, ws.cpu().numpy()[1024:1024 + REC_BYTES]


# g_mean 3: the tensor-core preparation; g_mean -3 (chunk decay near -190): the CUDA-core
# preparation of strongly decayed chunks (fp32, same record layout)
@pytest.mark.parametrize("g_mean", [3.0, -3.0])
@pytest.mark.parametrize("nrow", [64, 37])
def test_prep_record_matches_chunked_oracle(nrow, g_mean):
    inp, rec = _records(nrow, 300 + nrow, g_mean)
    f = lambda x: x[:, 0].double().numpy()
    T = chunked.chunk_tensors(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]),
                              inp["beta"][:, 0].double().numpy())
    n = nrow
    M_ref = -T["K_res"].T @ T["W"]
    P_ref = T["Q_dec"] - T["Aqk"] @ T["W"]
    # [M ; P]: two key-channel halves of 24 KB, each 192 K-major rows (M's 128, then P's 64)
    SB = [_sw128(rec[kb * 24576:(kb + 1) * 24576], 192) for kb in range(2)]
    M = np.concatenate([SB[kb][:128] for kb in range(2)], axis=1)
    P = np.concatenate([SB[kb][128:] for kb in range(2)], axis=1)
    # K_res: rows t, 64-column halves 8 KB apart; Aqk: K-major rows r
    K_res = np.concatenate([_sw128(rec[49152 + b * 8192:49152 + (b + 1) * 8192], 64) for b in range(2)], axis=1)
    Aqk = _sw128(rec[65536:73728], 64)
    U = np.concatenate([_sw64(rec[73728 + s * 4096:73728 + (s + 1) * 4096], 64) for s in range(4)], axis=1)
    gam = rec[90112:90624].copy().view(np.float32).astype(np.float64)

    def rel(a, b):
        return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)

    errs = {"M": rel(M, M_ref), "P": rel(P[:n], P_ref), "K_res": rel(K_res[:n], T["K_res"]),
            "U": rel(U[:n], T["U"]), "Aqk": rel(Aqk[:n, :n], T["Aqk"]),
            "B": rel(K_res[:n].T @ U[:n], T["K_res"].T @ T["U"]),
            "R": rel(Aqk[:n, :n] @ U[:n], T["Aqk"] @ T["U"]), "gamma": rel(gam, T["gamma"])}
    print("record errors nrow %d g_mean %g:" % (nrow, g_mean), {k: "%.2e" % v for k, v in errs.items()})
    # Bounds from the arithmetic: gamma is fp32 (a sum of 64 fp32 log-decays, one exp:
    # a few ulp, measured 2e-7); K_res, U, Aqk and P are bf16 images (one rounding of
    # relative 2^-9 per element, ~1.1e-3 in Frobenius norm, plus the rounding of the bf16
    # operands they are products of: measured 1.4e-3 to 2.8e-3); M = -K_res^T W and the
    # derived B and R are products of two rounded images (measured up to 3.9e-3).  About
    # 1.5x the largest measured error on either preparation.
    bound = {"gamma": 1e-6, "K_res": 5e-3, "U": 5e-3, "Aqk": 5e-3, "P": 5e-3, "M": 6e-3,
             "B": 6e-3, "R": 6e-3}
    for k, e in errs.items():
        assert e < bound[k], (k, e, bound[k])
    for x in (P[n:], K_res[n:], U[n:], Aqk[n:], Aqk[:, n:]):
        assert np.all(x == 0)
