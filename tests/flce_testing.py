"""Helpers shared by the GPU tests: move seeded numpy inputs to the GPU, run the
CUDA path through the C ABI binding, and compare with the oracle.

Tolerances: |d loss_i| <= 1e-3 and |d lse_i| <= 1e-3 absolute per token and
|d mean| / |mean| <= 1e-5, as required of the forward; the target logit gets
the same 1e-3 absolute bound (it is one fp32-accumulated dot product of
length D, with an error of order D * 2^-24 * sum_k |H_ik W_jk| << 1e-3 here).
"""
import numpy as np
import torch

LOSS_TOL = 1e-3
LSE_TOL = 1e-3
TARGET_TOL = 1e-3
MEAN_RTOL = 1e-5


def to_device(H, W, y, device="cuda:0"):
    def conv(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.to(device)
    return conv(H), conv(W), torch.from_numpy(np.ascontiguousarray(y, dtype=np.int64)).to(device)


def run(H, W, y, device="cuda:0", check=True):
    import linear_cross_entropy_bf16_b200 as flce
    Hd, Wd, yd = to_device(H, W, y, device)
    loss, lse, tgt, mean = flce.forward(Hd, Wd, yd, check=check)
    torch.cuda.synchronize()
    return {"loss": loss.cpu().numpy().astype(np.float64), "lse": lse.cpu().numpy().astype(np.float64),
            "target": tgt.cpu().numpy().astype(np.float64), "mean": float(mean.item())}


def compare(gpu, ref, rows=None, mean_ref=None):
    """Assert per-token parity on `rows` (indices into the GPU outputs; ref is indexed like rows)."""
    sel = slice(None) if rows is None else np.asarray(rows)
    for key, tol in (("loss", LOSS_TOL), ("lse", LSE_TOL), ("target", TARGET_TOL)):
        g = gpu[key][sel]
        d = np.abs(g - ref[key])
        assert np.all(np.isfinite(g)), f"{key}: non-finite GPU values"
        worst = int(np.argmax(d))
        assert d.max() <= tol, f"{key}: max |diff| {d.max():.3e} at sample {worst} (gpu {g[worst]!r}, oracle {ref[key][worst]!r})"
    if mean_ref is not None:
        assert abs(gpu["mean"] - mean_ref) <= MEAN_RTOL * abs(mean_ref), (gpu["mean"], mean_ref)
    return {k: float(np.abs(gpu[k][sel] - ref[k]).max()) for k in ("loss", "lse", "target")}


def check_properties(gpu, V):
    """Properties that hold at any size: finite, loss >= 0, lse >= target, mean = average."""
    import math
    assert np.all(np.isfinite(gpu["loss"])) and np.all(np.isfinite(gpu["lse"]))
    # the maximum's own term is exactly 1, so lse >= max z >= target logit: never negative
    assert np.all(gpu["loss"] >= 0.0)
    assert np.all(gpu["lse"] + LSE_TOL >= gpu["target"])
    # loss = lse - target logit, up to fp32 rounding of the stored lse
    assert np.all(np.abs(gpu["loss"] - (gpu["lse"] - gpu["target"])) <= 4e-7 * (1 + np.abs(gpu["lse"])) + 1e-6)
    m = math.fsum(gpu["loss"].tolist()) / len(gpu["loss"])
    assert abs(gpu["mean"] - m) <= 1e-6 * max(1.0, abs(m))
