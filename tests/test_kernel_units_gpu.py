"""Per-kernel parity of the tensor-core prep (steps a and b): the operand image
it writes for each (chunk, head) -- -W^T, Q e^G, Aqk^T, K e^{G_last - G},
T diag(beta) and e^{G_last} -- decoded from its 128-byte-swizzled bf16 layout and
compared quantity by quantity with the fp64 chunk equations of
tests/test_chunk_algebra.py on the same rounded inputs; and T (I + A) = I with
the fp64 A.  Covers full and partial chunks, KDA and the Gated DeltaNet prep."""
import numpy as np
import pytest
import torch

import workloads as W
from test_chunk_algebra import C, chunk_intra

pytestmark = pytest.mark.gpu

IMG_W, IMG_QG, IMG_B2, IMG_T, IMG_GAM = 0, 16384, 32768, 57344, 65536


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _sw(row, col):
    """Byte offset of element (row, col) in a 128-byte-swizzled tile of 64 bf16 per row."""
    return row * 128 + (((col >> 3) ^ (row & 7)) << 4) + (col & 7) * 2


def _bf16_at(img, offs):
    raw = img[offs[..., None] + np.arange(2)]                    # little-endian bf16 bytes
    u16 = raw[..., 0].astype(np.uint32) | (raw[..., 1].astype(np.uint32) << 8)
    return (u16 << 16).view(np.float32).astype(np.float64)


def decode(img):
    """One image (uint8 numpy) -> dict of fp64 matrices."""
    r = np.arange(C)[:, None]
    c = np.arange(128)[None, :]
    two_blocks = (c >> 6) * 8192 + np.vectorize(_sw)(r, c & 63)
    j = np.arange(C)[:, None]
    i = np.arange(C)[None, :]
    return {
        "W": -_bf16_at(img, IMG_W + np.vectorize(_sw)(c, r)),           # -W^T: [channel][token]
        "QG": _bf16_at(img, IMG_QG + two_blocks),
        "AqkT": _bf16_at(img, IMG_B2 + np.vectorize(_sw)(j, i)),          # [j][i] = Aqk[i][j]
        "KGl": _bf16_at(img, IMG_B2 + 8192 + two_blocks),
        "Tp": _bf16_at(img, IMG_T + np.vectorize(_sw)(r, np.arange(C)[None, :])),
        "gam": img[IMG_GAM:IMG_GAM + 512].view(np.float32).astype(np.float64),
    }


def _rel(a, b):
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a))


@pytest.mark.parametrize("gdn", [False, True])
def test_prep_image_matches_chunk_equations(kda, gdn):
    cfg = W.small_prefill(B=2, T=150, H=2, dk=128, dv=128, io_dtype="bf16", seed=90)
    inp = W.make_prefill(cfg, "cuda")
    log_a = W.scalar_gates(cfg.B, cfg.T, cfg.H, seed=90, device="cuda") if gdn else None
    g = log_a.unsqueeze(-1).expand(*log_a.shape, 128).contiguous() if gdn else inp["log_alpha"]
    imgs = kda.debug_prep_image(inp["q"], inp["k"], log_a if gdn else inp["log_alpha"], inp["beta"],
                                gate_scalar=gdn)
    torch.cuda.synchronize()
    imgs = imgs.cpu().numpy()
    h = lambda x: x.detach().cpu().double().numpy()
    q, k, gg, b = h(inp["q"]), h(inp["k"]), h(g), h(inp["beta"])
    nct = (cfg.T + C - 1) // C
    worst = {}
    for n in range(cfg.B):
        for ch in range(nct):
            t0 = ch * C
            L = min(C, cfg.T - t0)
            for hd in range(cfg.H):
                pad = lambda x: np.concatenate([x[n, t0:t0 + L, hd], np.zeros((C - L,) + x.shape[3:])])
                ref = chunk_intra(pad(q), pad(k), np.zeros((C, 128)), pad(gg),
                                  np.concatenate([b[n, t0:t0 + L, hd], np.zeros(C - L)]), 1.0)   # the image is unscaled
                got = decode(imgs[(n * nct + ch) * cfg.H + hd])
                bb = np.concatenate([b[n, t0:t0 + L, hd], np.zeros(C - L)])
                pairs = {"W": (got["W"], ref["W"]), "QG": (got["QG"], ref["QG"]),
                         "Aqk": (got["AqkT"].T, ref["Aqk"]), "KGl": (got["KGl"], ref["KGl"]),
                         "Tp": (got["Tp"], ref["T"] * bb[None, :]), "gam": (got["gam"], ref["gam"])}
                for name, (x, y) in pairs.items():
                    worst[name] = max(worst.get(name, 0.0), _rel(x, y))
                # T (I + A) = I on the rows and columns with beta > 0 (T' = T diag(beta))
                live = bb > 0
                Tg = np.zeros((C, C))
                Tg[:, live] = got["Tp"][:, live] / bb[live]
                resid = (Tg @ (np.eye(C) + ref["A"]))[np.ix_(live, live)] - np.eye(C)[np.ix_(live, live)]
                worst["T(I+A)-I"] = max(worst.get("T(I+A)-I", 0.0), float(np.abs(resid).max()))
    print("UNIT prep_image " + ("gdn " if gdn else "kda ") +
          " ".join(f"{k}={v:.2e}" for k, v in worst.items()))
    bar = {"W": 1e-2, "QG": 5e-3, "Aqk": 1e-2, "KGl": 5e-3, "Tp": 1e-2, "gam": 1e-5, "T(I+A)-I": 5e-2}
    for name, v in worst.items():
        assert v <= bar[name], (name, v)
