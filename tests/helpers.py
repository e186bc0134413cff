"""Shared test helpers: tolerances, error metric, device transfer."""
import numpy as np
import torch

# max relative error bounds for fp32 and bf16 inputs (fp32 state in both)
TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def slice_relerr(x, ref, lead: int) -> float:
    """max over the leading `lead` axes of max|x - ref| / max|ref| (per slice)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return 0.0
    xs = x.reshape(int(np.prod(x.shape[:lead])), -1)
    rs = ref.reshape(xs.shape)
    num = np.max(np.abs(xs - rs), axis=1)
    den = np.maximum(np.max(np.abs(rs), axis=1), 1e-30)
    err = num / den
    if not np.all(np.isfinite(x)):
        return float("inf")
    return float(np.max(err))


def m_err(m, ref) -> float:
    m = np.asarray(m, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if m.size == 0:
        return 0.0
    return float(np.max(np.abs(m - ref) / np.maximum(1.0, np.abs(ref))))


def dev(x, dtype=torch.float32):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def host(t):
    return None if t is None else t.detach().float().cpu().numpy()
