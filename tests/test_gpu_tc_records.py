"""White-box check of the tensor-core preparation kernel: decode the per-(chunk, head)
workspace record (shared-memory operand images, 128-byte swizzle) and compare every
chunk tensor with the fp64 chunked form of the oracle."""
import numpy as np
import pytest
import torch

from oracle import chunked
from linear_attention_rule_b200 import kda, synthetic
from tests.gpu_helpers import to_device

pytestmark = pytest.mark.gpu

REC_BYTES = 74240


def _sw128(img: np.ndarray, rows: int) -> np.ndarray:
    """bf16 image of `rows` rows x 64 elements, 128-byte swizzle -> float array."""
    b = img[: rows * 128].reshape(rows, 8, 16)
    out = np.empty((rows, 8, 16), dtype=np.uint8)
    for r in range(rows):
        for ch in range(8):
            out[r, ch] = b[r, ch ^ (r % 8)]
    return _bf16(out.reshape(rows, 128))


def _bf16(u8: np.ndarray) -> np.ndarray:
    u16 = u8.copy().view(np.uint16).astype(np.uint32) << 16
    return u16.view(np.float32).astype(np.float64)


def _records(nrow, seed):
    inp = synthetic.make_prefill_inputs([nrow], 1, 128, 128, torch.bfloat16, 3.0, 0.0, seed)
    d = to_device(inp)
    need = kda.kda_prefill_workspace_size(nrow, 1, 1, 128, 128, 64, torch.bfloat16)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty(nrow, 1, 128, dtype=torch.bfloat16, device="cuda")
    kda.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], out, C=64,
                    workspace=ws)
    assert kda.kda_get_device_status() == kda.KDA_OK
    rec = ws.cpu().numpy()[1024:1024 + REC_BYTES]
    return inp, rec


@pytest.mark.parametrize("nrow", [64, 37])
def test_prep_record_matches_chunked_oracle(nrow):
    inp, rec = _records(nrow, 300 + nrow)
    f = lambda x: x[:, 0].double().numpy()
    T = chunked.chunk_tensors(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]),
                              inp["beta"][:, 0].double().numpy())
    n = nrow
    Wt = _sw128(rec[0:16384], 128)            # [i][r] = W[r][i]
    Qt = _sw128(rec[16384:32768], 128)        # [i][r] = Q_dec[r][i]
    Kr = _sw128(rec[32768:49152], 128)        # [i][r] = K_res[r][i]
    Aq = _sw128(rec[49152:57344], 64)         # [r][s]
    Ut = _bf16(rec[57344:73728].reshape(128, 128))  # [j][r] = U[r][j]
    gam = rec[73728:74240].copy().view(np.float32).astype(np.float64)

    def rel(a, b):
        return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)

    errs = {
        "Q_dec": rel(Qt[:, :n].T, T["Q_dec"]),
        "K_res": rel(Kr[:, :n].T, T["K_res"]),
        "Aqk": rel(Aq[:n, :n], T["Aqk"]),
        "W": rel(Wt[:, :n].T, T["W"]),
        "U": rel(Ut[:, :n].T, T["U"]),
        "gamma": rel(gam, T["gamma"]),
    }
    print(nrow, {k: "%.2e" % v for k, v in errs.items()})
    for k, e in errs.items():
        assert e < 1e-2, (k, e)
    # padded rows are exactly zero
    assert np.all(Qt[:, n:] == 0) and np.all(Wt[:, n:] == 0) and np.all(Ut[:, n:] == 0)
    assert np.all(Aq[n:, :] == 0)
