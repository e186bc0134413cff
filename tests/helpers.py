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


def _denominators(q, k, igate, fgate, n0, m0, num_blocks):
    """fp64 per token [B, NH, nb, S]: den_t = max(|n'_t . q_t|, e^{-m_t}) and the same with the
    absolute values |n'_abs| . |q_t| (n'_abs the normaliser of |k| and |n0|, same gates)."""
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
    na = np.abs(n)
    m = np.zeros((B, NH)) if m0 is None else np.asarray(m0, np.float64).reshape(B, NH)
    den = np.zeros((B, NH, num_blocks, S))
    den_abs = np.zeros((B, NH, num_blocks, S))
    for t in range(S):
        m_new = np.maximum(lf[:, :, t] + m, ig[:, :, t])
        fp = np.exp(lf[:, :, t] + m - m_new)[..., None, None]
        ip = np.exp(ig[:, :, t] - m_new)[..., None, None]
        n = fp * n + ip * kb[:, :, t]
        na = fp * na + ip * np.abs(kb[:, :, t])
        m = m_new
        floor = np.exp(-m)[..., None]
        den[..., t] = np.maximum(np.abs(np.sum(n * qb[:, :, t], -1)), floor)
        den_abs[..., t] = np.maximum(np.sum(na * np.abs(qb[:, :, t]), -1), floor)
    return den, den_abs


def readout_scale(q, k, v, igate, fgate, C0=None, n0=None, m0=None, num_blocks: int = 1):
    """What rounding the recurrence's terms can do to h, fp64: returns (kappa [B, NH, nb, S],
    h_abs [B, NH, S, DHV]).  h_t = num_t / den_t with num_t = C'_t q_t and den_t =
    max(|n'_t . q_t|, e^{-m_t}); if every element of the state (and of the intra-chunk terms)
    carries a relative error delta, then

        |d num_t,i| <= delta sum_j |C'_t,ij q_t,j| <= delta num_abs_t,i,
        |d den_t|   <= delta sum_j |n'_t,j q_t,j|  <= delta den_abs_t,

    where num_abs, den_abs are the same recurrence run on |q|, |k|, |v|, |C0|, |n0| (all gate
    weights are positive).  With kappa_t = den_abs_t / den_t and h_abs = num_abs / den_abs (the
    read-out of that absolute run):

        |d h_t,i| <= delta (num_abs_t,i + |h_t,i| den_abs_t) / den_t
                  =  delta kappa_t (h_abs_t,i + |h_t,i|).

    With q and k of both signs, num and den can cancel, so kappa_t is unbounded and no
    fixed-precision evaluation meets a fixed relative error on such tokens.  Used only to scale
    a tolerance, never as an expected value.
    """
    import oracle
    den, den_abs = _denominators(q, k, igate, fgate, n0, m0, num_blocks)
    a = lambda x: None if x is None else np.abs(x)
    h_abs = oracle.sequential(a(q), a(k), a(v), igate, fgate, None, a(C0), a(n0), m0, num_blocks=num_blocks)[0]
    return den_abs / den, np.abs(h_abs)


def conditioned_excess(h, ref, kappa, h_abs, tol: float, delta: float) -> float:
    """Largest ratio, over tokens and values, of an element's error |h_t,i - ref_t,i| to its
    bound tol * max_i |ref_t,i| + delta * kappa_t * (h_abs_t,i + |ref_t,i|) (kappa, h_abs from
    readout_scale); <= 1 passes.  The first term is the fixed tolerance relative to the token's
    own read-out (stricter than relative to the whole slice, which one huge token of a slice
    would make lenient on all the others), the second what a relative error delta in the terms
    costs a token whose read-out cancels."""
    h = np.asarray(h, np.float64)
    ref = np.asarray(ref, np.float64)
    B, NH, S, DHV = ref.shape
    nb = kappa.shape[2]
    split = lambda x: np.asarray(x, np.float64).reshape(B, NH, S, nb, DHV // nb).transpose(0, 1, 3, 2, 4)
    hb, rb, ab = split(h), split(ref), split(h_abs)
    if not np.all(np.isfinite(hb)):
        return float("inf")
    tok = np.max(np.abs(rb), axis=-1, keepdims=True)            # [B, NH, nb, S, 1]
    bound = tol * tok + delta * kappa[..., None] * (ab + np.abs(rb))
    return float(np.max(np.abs(hb - rb) / np.maximum(bound, 1e-300)))


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
