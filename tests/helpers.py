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


def denominator_condition(q, k, igate, fgate, n0=None, m0=None, num_blocks: int = 1):
    """Condition number of each token's read-out denominator, fp64, [B, NH, nb, S]:

        kappa_t = sum_i |n'_{t,i} q_{t,i}| / max(|n'_t . q_t|, exp(-m_t)).

    A relative error delta in the terms of n'.q (rounding of n' and of the dot product)
    moves the denominator by at most delta * kappa_t of itself, and h_t by the same
    factor.  With q and k of both signs n'.q can cancel, so kappa_t is unbounded and no
    fixed-precision evaluation keeps a fixed relative error on such a token.  Used only to
    scale a tolerance, never as an expected value.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    ig = np.asarray(igate, np.float64)
    fg = np.asarray(fgate, np.float64)
    B, NH, S, D = q.shape
    dk = D // num_blocks
    qb = q.reshape(B, NH, S, num_blocks, dk)
    kb = k.reshape(B, NH, S, num_blocks, dk)
    lf = np.minimum(fg, 0.0) - np.log1p(np.exp(-np.abs(fg)))
    n = np.zeros((B, NH, num_blocks, dk)) if n0 is None else np.asarray(n0, np.float64).reshape(B, NH, num_blocks, dk)
    m = np.zeros((B, NH)) if m0 is None else np.asarray(m0, np.float64).reshape(B, NH)
    out = np.zeros((B, NH, num_blocks, S))
    for t in range(S):
        m_new = np.maximum(lf[:, :, t] + m, ig[:, :, t])
        fp = np.exp(lf[:, :, t] + m - m_new)[..., None, None]
        ip = np.exp(ig[:, :, t] - m_new)[..., None, None]
        n = fp * n + ip * kb[:, :, t]
        m = m_new
        prod = n * qb[:, :, t]
        out[..., t] = np.sum(np.abs(prod), -1) / np.maximum(np.abs(np.sum(prod, -1)), np.exp(-m)[..., None])
    return out


def conditioned_excess(h, ref, kappa, tol: float, delta: float) -> float:
    """Largest ratio, over (batch, head, block) slices and tokens, of a token's error to its
    bound tol * max|ref of the slice| + delta * kappa_t * max|ref_t|; <= 1 passes.

    h, ref [B, NH, S, DHV] (DHV split into nb blocks as kappa's third axis); kappa from
    denominator_condition.  The first term is the fixed tolerance of the comparison, the
    second what a relative error delta in the denominator's terms costs a token whose
    denominator cancels (see denominator_condition).
    """
    h = np.asarray(h, np.float64)
    ref = np.asarray(ref, np.float64)
    B, NH, S, DHV = ref.shape
    nb = kappa.shape[2]
    hb = h.reshape(B, NH, S, nb, DHV // nb).transpose(0, 1, 3, 2, 4)
    rb = ref.reshape(B, NH, S, nb, DHV // nb).transpose(0, 1, 3, 2, 4)
    if not np.all(np.isfinite(hb)):
        return float("inf")
    err = np.max(np.abs(hb - rb), -1)                         # [B, NH, nb, S]
    tok = np.max(np.abs(rb), -1)                              # [B, NH, nb, S]
    scale = np.max(tok, -1, keepdims=True)                    # [B, NH, nb, 1]
    bound = tol * np.maximum(scale, 1e-30) + delta * kappa * tok
    return float(np.max(err / bound))


class Guarded:
    """A device output tensor with guard bands on both sides: the tensor is a view into the
    middle of a larger byte buffer whose `guard` bytes before and after it hold a fixed
    pattern.  ``intact()`` tells whether a kernel wrote outside the tensor (a store past a
    ragged tail, a wrong stride or offset).  Standing in for a memory checker, which this
    setting does not offer."""

    FILL = 0xA5

    def __init__(self, shape, dtype, guard: int = 4096):
        n = 1
        for d in shape:
            n *= int(d)
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.guard = guard
        self.buf = torch.full((2 * guard + self.nbytes,), self.FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[guard:guard + self.nbytes].view(dtype).view(tuple(int(d) for d in shape))

    def fill(self, x: torch.Tensor):
        self.t.copy_(x)
        return self.t

    def intact(self) -> bool:
        g, n = self.guard, self.nbytes
        return bool((self.buf[:g] == self.FILL).all().item()) and bool((self.buf[g + n:] == self.FILL).all().item())


def guarded_like(shape, dtype, n=1):
    return [Guarded(shape, dtype) for _ in range(n)]
