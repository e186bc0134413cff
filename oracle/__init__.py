"""fp64 CPU oracle for the mLSTM / retention recurrence -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it, and it imports nothing from them: the two sides share only
the seeded input generators, which hold none of the method's arithmetic.

Contents
--------
``sequential``       C, fp64, one token at a time (``mlstm_oracle.c``).  The
                     primary oracle; also the timed CPU baseline.
``parallel_form``    numpy, fp64, the quadratic "parallel" evaluation with the
                     decay matrix D (Edifice.Attention.RetNet, "Key Innovation",
                     generalised to the mLSTM's stabilised gates).  Tiny inputs.
``chunkwise``        numpy, fp64, the chunked evaluation (intra-chunk quadratic
                     part plus an inter-chunk carried state), used to check the
                     chunk algebra independently of any GPU code.
``unstabilised``     numpy, fp64, the recurrence with raw exponential gates and
                     the floor 1 of the mLSTM read-out, no stabiliser at all.
``state_bytes``      size of a model's recurrent state (xLSTM 7B "Modelled costs").
``sequential_scalar_normaliser``  numpy, fp64, the variant with a scalar normaliser and a
                     learnable bias (Edifice.Recurrent.XLSTMv2, "Key Improvements" #2).
``theta_rotate``, ``group_norm_gate``, ``retention_block``  numpy, fp64, the steps
                     either side of retention (Edifice.Attention.RetNet): the rotation of
                     q and k, the per-head GroupNorm and the SiLU gate, and their composition.
``gdn2_sequential``, ``gdn2_chunk``  numpy, fp64, Gated DeltaNet-2 (burn-gdn2): the
                     token-by-token recurrence and its chunked (triangular-solve) evaluation.
``sequential_backward``  numpy, fp64, gradients of ``sequential`` by reverse-mode
                     differentiation of its steps in reverse order (backpropagation
                     through time); pinned by central finite differences.

Pins (tests/test_oracle_*.py) tie every function to something other than
itself: closed forms, brute-force double loops, special cases and invariants.
The per-block normaliser (num_blocks > 1) and the optional output gate o_t are
fixed by this project's reading of the pages, not by them: parity unpinned
for those two readings (their self-consistency is still tested).  Likewise for
the NEXT-row readings: the frequencies of Theta (theta_j = base^{-2j/D} on
interleaved pairs; the pins fix the rotation's form and its relative-position
property, not the frequency choice), and the GDN-2 update beyond what the page
states (the pins fix the per-channel roles of the erase and write gates and the
delta-rule property of the KDA reduction it names; the order decay -> erase ->
write and the erase vector b o k are readings): parity unpinned by the pages
for those parts.  GroupNorm and SiLU are pinned by torch's routines.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlstm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile mlstm_oracle.c with gcc into oracle/liboracle.so (in-tree)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_mlstm_sequential.argtypes = [I] * 7 + [P] * 13 + [I]
        _lib.oracle_mlstm_sequential.restype = I
    return _lib


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def sequential(q, k, v, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None,
               num_blocks: int = 1, retention: bool = False, threads: int | None = None):
    """Sequential fp64 recurrence (mlstm_oracle.c).

    q, k: [B,NH,S,DHQK]; v: [B,NH,S,DHV]; igate, fgate: [B,NH,S] pre-activations;
    ogate: [B,NH,S,DHV] already-activated output gate or None (= 1);
    C0: [B,NH,nb,DHV/nb,DHQK/nb]; n0: [B,NH,nb,DHQK/nb]; m0: [B,NH]; None = zeros.
    Returns (h, C, n, m); n and m are None in retention mode.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = int(num_blocks)
    if DHQK % nb or DHV % nb:
        raise ValueError("num_blocks must divide DHQK and DHV")
    dk, dv = DHQK // nb, DHV // nb
    ig, fg = _f64(igate), _f64(fgate)
    og = _f64(ogate)
    C0, n0, m0 = _f64(C0), _f64(n0), _f64(m0)
    h = np.zeros((B, NH, S, DHV))
    C = np.zeros((B, NH, nb, dv, dk))
    n = None if retention else np.zeros((B, NH, nb, dk))
    m = None if retention else np.zeros((B, NH))
    if threads is None:
        threads = len(os.sched_getaffinity(0))
    rc = lib.oracle_mlstm_sequential(B, NH, S, DHQK, DHV, nb, int(bool(retention)),
                                     _ptr(q), _ptr(k), _ptr(v), _ptr(ig), _ptr(fg), _ptr(og),
                                     _ptr(C0), _ptr(n0), _ptr(m0),
                                     _ptr(h), _ptr(C), _ptr(n), _ptr(m), int(threads))
    if rc != 0:
        raise ValueError("oracle_mlstm_sequential rejected the shapes")
    return h, C, n, m


def log_sigmoid(x):
    """log(1 / (1 + exp(-x))) in the overflow-free form min(x, 0) - log1p(exp(-|x|))."""
    x = np.asarray(x, dtype=np.float64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def retention_gamma(NH: int):
    """Per-head decay gamma_h = 1 - 2^(-5-h), h = 0 .. NH-1 (RetNet "Multi-Scale Retention")."""
    return 1.0 - np.exp2(-5.0 - np.arange(NH, dtype=np.float64))


def _split_blocks(x, nb):
    """[..., D] -> [..., nb, D/nb] (block j takes the j-th contiguous slice)."""
    return x.reshape(x.shape[:-1] + (nb, x.shape[-1] // nb))


def parallel_form(q, k, v, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None,
                  num_blocks: int = 1, retention: bool = False):
    """Quadratic (all pairs) evaluation, fp64.  For tiny S only.

    Retention (RetNet "Key Innovation"): Y = (Q K^T * D) V with
    D[t, s] = gamma^(t-s) for s <= t, plus the initial state decayed by gamma^(t+1).
    mLSTM: log D[t, s] = b_t - b_s + itilde_s (s <= t) with b the inclusive cumulative
    sum of log f; the initial state enters with weight b_t + m0; the stabiliser is the
    row maximum of those log weights, which is the recurrence's m_t.
    Returns (h, C, n, m) like ``sequential``.
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = num_blocks
    dk, dv = DHQK // nb, DHV // nb
    qb = _split_blocks(q, nb).transpose(0, 1, 3, 2, 4)  # [B,NH,nb,S,dk]
    kb = _split_blocks(k, nb).transpose(0, 1, 3, 2, 4)
    vb = _split_blocks(v, nb).transpose(0, 1, 3, 2, 4)  # [B,NH,nb,S,dv]
    C0 = np.zeros((B, NH, nb, dv, dk)) if C0 is None else np.asarray(C0, dtype=np.float64)
    n0 = np.zeros((B, NH, nb, dk)) if n0 is None else np.asarray(n0, dtype=np.float64)
    m0 = np.zeros((B, NH)) if m0 is None else np.asarray(m0, dtype=np.float64)
    tril = np.tril(np.ones((S, S), dtype=bool))
    t_idx = np.arange(S)
    h = np.zeros((B, NH, nb, S, dv))
    C = np.zeros((B, NH, nb, dv, dk))
    n = np.zeros((B, NH, nb, dk))
    m = np.zeros((B, NH))
    gam = retention_gamma(NH)
    for b in range(B):
        for hd in range(NH):
            if retention:
                g = gam[hd]
                expo = (t_idx[:, None] - t_idx[None, :]).astype(np.float64)
                D = np.where(tril, g ** np.where(tril, expo, 0.0), 0.0)
                w_init = g ** (t_idx + 1.0)
                for j in range(nb):
                    Q, K, V = qb[b, hd, j], kb[b, hd, j], vb[b, hd, j]
                    h[b, hd, j] = (Q @ K.T * D) @ V + w_init[:, None] * (Q @ C0[b, hd, j].T)
                    wS = g ** (S - 1 - t_idx)
                    C[b, hd, j] = (V * wS[:, None]).T @ K + g ** S * C0[b, hd, j]
                continue
            lf = log_sigmoid(fgate[b, hd])
            li = np.asarray(igate[b, hd], dtype=np.float64)
            bcum = np.cumsum(lf)
            logD = np.where(tril, bcum[:, None] - bcum[None, :] + li[None, :], -np.inf)
            log_init = bcum + m0[b, hd]
            mt = np.maximum(log_init, logD.max(axis=1))
            D = np.exp(logD - mt[:, None])
            w_init = np.exp(log_init - mt)
            # final state at t = S-1
            mS = mt[-1] if S > 0 else m0[b, hd]
            wS = np.exp(bcum[-1] - bcum + li - mS) if S > 0 else np.zeros(0)
            aS = np.exp(bcum[-1] + m0[b, hd] - mS) if S > 0 else 1.0
            for j in range(nb):
                Q, K, V = qb[b, hd, j], kb[b, hd, j], vb[b, hd, j]
                P = (Q @ K.T) * D
                num = P @ V + w_init[:, None] * (Q @ C0[b, hd, j].T)
                den = P.sum(axis=1) + w_init * (Q @ n0[b, hd, j])
                hh = num / np.maximum(np.abs(den), np.exp(-mt))[:, None]
                if ogate is not None:
                    hh = hh * _split_blocks(np.asarray(ogate[b, hd], dtype=np.float64), nb)[:, j, :]
                h[b, hd, j] = hh
                C[b, hd, j] = (V * wS[:, None]).T @ K + aS * C0[b, hd, j]
                n[b, hd, j] = (K * wS[:, None]).sum(axis=0) + aS * n0[b, hd, j]
            m[b, hd] = mS
    h = h.transpose(0, 1, 3, 2, 4).reshape(B, NH, S, DHV)
    if retention:
        return h, C, None, None
    return h, C, n, m


def chunkwise(q, k, v, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None,
              num_blocks: int = 1, retention: bool = False, chunk: int = 16):
    """Chunked evaluation, fp64: quadratic inside each chunk, a carried state between.

    Per chunk with local cumulative log-forget b (inclusive) and total g:
      m_t   = max(b_t + m_c, max_{s<=t} (b_t - b_s + itilde_s))   (max-plus form of the
              stabiliser recurrence)
      h_t   = [sum_s e^{b_t-b_s+i_s-m_t} (q_t.k_s) v_s + e^{b_t+m_c-m_t} C_c q_t] / den_t
      C_c+1 = e^{g+m_c-m_c+1} C_c + sum_s e^{g-b_s+i_s-m_c+1} v_s k_s^T
    Retention uses gamma powers and no normaliser.  S need not divide by chunk.
    Returns (h, C, n, m) like ``sequential``.
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = num_blocks
    dk, dv = DHQK // nb, DHV // nb
    qb = _split_blocks(q, nb)
    kb = _split_blocks(k, nb)
    vb = _split_blocks(v, nb)
    ob = None if ogate is None else _split_blocks(np.asarray(ogate, dtype=np.float64), nb)
    C = np.zeros((B, NH, nb, dv, dk)) if C0 is None else np.array(C0, dtype=np.float64)
    n = np.zeros((B, NH, nb, dk)) if n0 is None else np.array(n0, dtype=np.float64)
    m = np.zeros((B, NH)) if m0 is None else np.array(m0, dtype=np.float64)
    h = np.zeros((B, NH, S, nb, dv))
    gam = retention_gamma(NH)
    for b in range(B):
        for hd in range(NH):
            for c0 in range(0, S, chunk):
                L = min(chunk, S - c0)
                sl = slice(c0, c0 + L)
                tril = np.tril(np.ones((L, L), dtype=bool))
                if retention:
                    lf = np.full(L, np.log(gam[hd]))
                    li = np.zeros(L)
                else:
                    lf = log_sigmoid(fgate[b, hd, sl])
                    li = np.asarray(igate[b, hd, sl], dtype=np.float64)
                bl = np.cumsum(lf)
                g = bl[-1]
                logD = np.where(tril, bl[:, None] - bl[None, :] + li[None, :], -np.inf)
                mc = 0.0 if retention else m[b, hd]
                if retention:
                    mt = np.zeros(L)
                else:
                    mt = np.maximum(bl + mc, logD.max(axis=1))
                D = np.exp(logD - mt[:, None])
                s_inter = np.exp(bl + mc - mt)
                m_next = 0.0 if retention else mt[-1]
                a = np.exp(g + mc - m_next)
                w = np.exp(g - bl + li - m_next)
                for j in range(nb):
                    Q, K, V = qb[b, hd, sl, j], kb[b, hd, sl, j], vb[b, hd, sl, j]
                    P = (Q @ K.T) * D
                    num = P @ V + s_inter[:, None] * (Q @ C[b, hd, j].T)
                    if retention:
                        hh = num
                    else:
                        den = P.sum(axis=1) + s_inter * (Q @ n[b, hd, j])
                        hh = num / np.maximum(np.abs(den), np.exp(-mt))[:, None]
                        if ob is not None:
                            hh = hh * ob[b, hd, sl, j]
                        n[b, hd, j] = a * n[b, hd, j] + (K * w[:, None]).sum(axis=0)
                    h[b, hd, sl, j] = hh
                    C[b, hd, j] = a * C[b, hd, j] + (V * w[:, None]).T @ K
                if not retention:
                    m[b, hd] = m_next
    h = h.reshape(B, NH, S, DHV)
    if retention:
        return h, C, None, None
    return h, C, n, m


def unstabilised(q, k, v, igate, fgate, ogate=None, C0=None, n0=None, num_blocks: int = 1):
    """The mLSTM recurrence with raw gates i = exp(itilde), f = sigmoid(ftilde), fp64.

    C_t = f C + i v k^T, n_t = f n + i k, h_t = o * C_t q_t / max(|n_t . q_t|, 1); no
    stabiliser.  Valid only while exp(itilde) and the products stay in range.
    Returns (h, C_true, n_true) with the state in raw (unstabilised) units.
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = num_blocks
    dk, dv = DHQK // nb, DHV // nb
    qb, kb, vb = _split_blocks(q, nb), _split_blocks(k, nb), _split_blocks(v, nb)
    C = np.zeros((B, NH, nb, dv, dk)) if C0 is None else np.array(C0, dtype=np.float64)
    n = np.zeros((B, NH, nb, dk)) if n0 is None else np.array(n0, dtype=np.float64)
    h = np.zeros((B, NH, S, nb, dv))
    f = 1.0 / (1.0 + np.exp(-np.asarray(fgate, dtype=np.float64)))
    i = np.exp(np.asarray(igate, dtype=np.float64))
    for t in range(S):
        ft = f[:, :, t, None, None, None]
        it = i[:, :, t, None, None, None]
        C = ft * C + it * vb[:, :, t, :, :, None] * kb[:, :, t, :, None, :]
        n = f[:, :, t, None, None] * n + i[:, :, t, None, None] * kb[:, :, t]
        num = np.einsum("bhjvk,bhjk->bhjv", C, qb[:, :, t])
        den = np.maximum(np.abs(np.einsum("bhjk,bhjk->bhj", n, qb[:, :, t])), 1.0)
        ht = num / den[..., None]
        if ogate is not None:
            ht = ht * _split_blocks(np.asarray(ogate[:, :, t], dtype=np.float64), nb)
        h[:, :, t] = ht
    return h.reshape(B, NH, S, DHV), C, n


def sequential_scalar_normaliser(q, k, v, igate, fgate, bias, ogate=None, C0=None, n0=None, m0=None,
                                  num_blocks: int = 1):
    """The mLSTM with the normaliser of Edifice.Recurrent.XLSTMv2 "Key Improvements" #2: a
    scalar n_t = f_t n_{t-1} + i_t (no key vector) and a learnable bias in the denominator,
    h_t = o_t * (C_t q_t) / max(|n_t + bias|, 1), fp64, one token at a time.  Gates and their
    stabiliser as in ``sequential``; in stabilised units n'_t = f' n'_{t-1} + i' and the
    denominator is max(|n'_t + bias e^{-m_t}|, e^{-m_t}).  n is per head (it depends on the
    gates only, so the blocks of a head share it).

    bias: [NH]; n0: [B,NH] stabilised; other arguments as for ``sequential``.
    Returns (h, C, n [B,NH], m [B,NH]).
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = num_blocks
    dk, dv = DHQK // nb, DHV // nb
    C0 = np.zeros((B, NH, nb, dv, dk)) if C0 is None else np.asarray(C0, dtype=np.float64)
    n0 = np.zeros((B, NH)) if n0 is None else np.asarray(n0, dtype=np.float64)
    m0 = np.zeros((B, NH)) if m0 is None else np.asarray(m0, dtype=np.float64)
    bias = np.asarray(bias, dtype=np.float64)
    h = np.zeros((B, NH, S, DHV))
    C = np.zeros((B, NH, nb, dv, dk))
    n = np.zeros((B, NH))
    m = np.zeros((B, NH))
    for b in range(B):
        for hd in range(NH):
            Cs = [C0[b, hd, j].copy() for j in range(nb)]
            ns, mt = n0[b, hd], m0[b, hd]
            for t in range(S):
                lf = float(log_sigmoid(fgate[b, hd, t]))
                li = float(igate[b, hd, t])
                m_new = max(lf + mt, li)
                fp, ip = math.exp(lf + mt - m_new), math.exp(li - m_new)
                mt = m_new
                ns = fp * ns + ip
                den = max(abs(ns + bias[hd] * math.exp(-mt)), math.exp(-mt))
                for j in range(nb):
                    sk, sv = slice(j * dk, (j + 1) * dk), slice(j * dv, (j + 1) * dv)
                    Cs[j] = fp * Cs[j] + ip * np.outer(v[b, hd, t, sv], k[b, hd, t, sk])
                    ht = Cs[j] @ q[b, hd, t, sk] / den
                    if ogate is not None:
                        ht = ht * np.asarray(ogate[b, hd, t, sv], dtype=np.float64)
                    h[b, hd, t, sv] = ht
            for j in range(nb):
                C[b, hd, j] = Cs[j]
            n[b, hd], m[b, hd] = ns, mt
    return h, C, n, m


def sequential_backward(q, k, v, dh, igate=None, fgate=None, ogate=None, C0=None, n0=None, m0=None,
                        dC=None, dn=None, num_blocks: int = 1, retention: bool = False):
    """Gradients of the sequential recurrence, fp64: its steps differentiated in reverse order.

    The forward step (mLSTM "Core idea", gates stabilised in log space) is
        lf = logsigmoid(ftilde);  m_t = max(lf + m_{t-1}, itilde_t)
        f' = exp(lf + m_{t-1} - m_t);  i' = exp(itilde_t - m_t)
        C'_t = f' C'_{t-1} + i' v_t k_t^T;  n'_t = f' n'_{t-1} + i' k_t
        h_t = o_t * (C'_t q_t) / max(|n'_t . q_t|, exp(-m_t))
    (retention: f' = gamma_h, i' = 1, h_t = C'_t q_t).  h does not depend on the stabiliser:
    with C'_t = exp(-m_t) C_t the division removes exp(-m_t) for any sequence m, so the steps
    are differentiated with m held at its forward values and the result is the exact gradient.
    The returned final state (C'_S, n'_S) is differentiated with m_S held fixed as well (dC, dn
    are the gradients of a loss on exp(m_S) C'_S, n'_S written in stabilised units); the
    initial state enters as exp(m0) C0, so dm0 = <dC0, C0> + dn0 . n0.

    dh: [B,NH,S,DHV]; dC: [B,NH,nb,dv,dk]; dn: [B,NH,nb,dk] (None = 0).
    Returns dict(dq, dk, dv, di, df, do, dC0, dn0, dm0); di, df, dn0, dm0 are None in retention
    mode, do is None without an output gate (or in retention mode).
    """
    q, k, v, dh = (np.asarray(a, dtype=np.float64) for a in (q, k, v, dh))
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    nb = num_blocks
    dk, dv = DHQK // nb, DHV // nb
    use_o = ogate is not None and not retention
    og = np.asarray(ogate, dtype=np.float64) if use_o else None
    C0 = np.zeros((B, NH, nb, dv, dk)) if C0 is None else np.asarray(C0, dtype=np.float64)
    n0 = np.zeros((B, NH, nb, dk)) if n0 is None else np.asarray(n0, dtype=np.float64)
    m0 = np.zeros((B, NH)) if m0 is None else np.asarray(m0, dtype=np.float64)
    dCS = np.zeros((B, NH, nb, dv, dk)) if dC is None else np.asarray(dC, dtype=np.float64)
    dnS = np.zeros((B, NH, nb, dk)) if dn is None else np.asarray(dn, dtype=np.float64)
    gam = retention_gamma(NH)
    out = {key: np.zeros_like(x) for key, x in (("dq", q), ("dk", k), ("dv", v))}
    out["do"] = np.zeros_like(dh) if use_o else None
    out["dC0"] = np.zeros((B, NH, nb, dv, dk))
    di = np.zeros((B, NH, S)) if not retention else None
    df = np.zeros((B, NH, S)) if not retention else None
    dn0 = np.zeros((B, NH, nb, dk)) if not retention else None
    dm0 = np.zeros((B, NH)) if not retention else None
    for b in range(B):
        for hd in range(NH):
            # gate quantities shared by the blocks of the head
            if retention:
                fp = np.full(S, gam[hd])
                ip = np.ones(S)
                mt = np.zeros(S)
            else:
                lf = log_sigmoid(fgate[b, hd])
                li = np.asarray(igate[b, hd], dtype=np.float64)
                mt = np.zeros(S)
                mprev = m0[b, hd]
                fp = np.zeros(S)
                ip = np.zeros(S)
                for t in range(S):
                    mt[t] = max(lf[t] + mprev, li[t])
                    fp[t] = math.exp(lf[t] + mprev - mt[t])
                    ip[t] = math.exp(li[t] - mt[t])
                    mprev = mt[t]
            dlf = np.zeros(S)
            dli = np.zeros(S)
            for j in range(nb):
                sk, sv = slice(j * dk, (j + 1) * dk), slice(j * dv, (j + 1) * dv)
                Q, K, V = q[b, hd, :, sk], k[b, hd, :, sk], v[b, hd, :, sv]
                dH = dh[b, hd, :, sv]
                O = og[b, hd, :, sv] if use_o else np.ones((S, dv))
                # forward, keeping every state
                Cs = np.zeros((S + 1, dv, dk))
                ns = np.zeros((S + 1, dk))
                Cs[0], ns[0] = C0[b, hd, j], n0[b, hd, j]
                num = np.zeros((S, dv))
                dd = np.zeros(S)
                den = np.ones(S)
                for t in range(S):
                    Cs[t + 1] = fp[t] * Cs[t] + ip[t] * np.outer(V[t], K[t])
                    ns[t + 1] = fp[t] * ns[t] + ip[t] * K[t]
                    num[t] = Cs[t + 1] @ Q[t]
                    if not retention:
                        dd[t] = ns[t + 1] @ Q[t]
                        den[t] = max(abs(dd[t]), math.exp(-mt[t]))
                # backward, t = S-1 .. 0; D, G: gradients of C'_t, n'_t accumulated so far
                D = dCS[b, hd, j].copy()
                G = dnS[b, hd, j].copy()
                for t in range(S - 1, -1, -1):
                    # h_t = o * num_t / den_t
                    dnum = O[t] * dH[t] / den[t]
                    if use_o:
                        out["do"][b, hd, t, sv] = dH[t] * num[t] / den[t]
                    ddd = 0.0
                    if not retention and abs(dd[t]) > math.exp(-mt[t]):
                        dden = -np.sum(O[t] * dH[t] * num[t]) / den[t] ** 2
                        ddd = dden * math.copysign(1.0, dd[t])
                    # num_t = C'_t q_t, d_t = n'_t . q_t
                    D = D + np.outer(dnum, Q[t])
                    G = G + ddd * Q[t]
                    out["dq"][b, hd, t, sk] = Cs[t + 1].T @ dnum + ddd * ns[t + 1]
                    # C'_t = f' C'_{t-1} + i' v k^T, n'_t = f' n'_{t-1} + i' k
                    out["dv"][b, hd, t, sv] = ip[t] * (D @ K[t])
                    out["dk"][b, hd, t, sk] = ip[t] * (D.T @ V[t]) + (0.0 if retention else ip[t]) * G
                    if not retention:
                        dip = V[t] @ D @ K[t] + G @ K[t]
                        dfp = np.sum(D * Cs[t]) + G @ ns[t]
                        dli[t] += ip[t] * dip  # d i'/d itilde = i'
                        dlf[t] += fp[t] * dfp  # d f'/d lf = f'
                    D = fp[t] * D
                    G = fp[t] * G
                out["dC0"][b, hd, j] = D
                if not retention:
                    dn0[b, hd, j] = G
                    dm0[b, hd] += np.sum(D * C0[b, hd, j]) + G @ n0[b, hd, j]
            if not retention:
                di[b, hd] = dli
                # d logsigmoid(x)/dx = sigmoid(-x)
                df[b, hd] = dlf / (1.0 + np.exp(np.asarray(fgate[b, hd], dtype=np.float64)))
    out.update(di=di, df=df, dn0=dn0, dm0=dm0)
    return out


def theta_rotate(x, pos0=None, base: float = 10000.0):
    """The relative-position rotation Theta that RetNet applies to queries and keys before
    retention (Edifice.Attention.RetNet, "Key Innovation": Y = (Q Theta) D (K Theta)^T V),
    fp64.  Theta is not spelled out on the page; the reading built here is the complex form
    Theta_n = e^{i n theta}: the head vector's entries (2j, 2j+1) are one complex number,
    multiplied by e^{i p theta_j} at sequence position p, theta_j = base^{-2j/D}.  The same
    rotation on q and k makes (Q Theta)(K Theta)^T depend on positions only through n - m.

    x: [B,NH,S,D], D even; pos0: [B] position of token 0 of each sequence (None = 0).
    Returns the rotated x, fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    B, NH, S, D = x.shape
    pos0 = np.zeros(B, dtype=np.int64) if pos0 is None else np.asarray(pos0, dtype=np.int64)
    theta = base ** (-2.0 * np.arange(D // 2) / D)
    out = np.empty_like(x)
    for b in range(B):
        pos = (pos0[b] + np.arange(S)).astype(np.float64)
        ang = pos[:, None] * theta[None, :]                # [S, D/2]
        c, s_ = np.cos(ang), np.sin(ang)
        x0, x1 = x[b, :, :, 0::2], x[b, :, :, 1::2]        # [NH, S, D/2]
        out[b, :, :, 0::2] = x0 * c - x1 * s_
        out[b, :, :, 1::2] = x0 * s_ + x1 * c
    return out


def silu(x):
    """x sigmoid(x), fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def group_norm_gate(h, g=None, weight=None, bias=None, eps: float = 1e-5):
    """Per-head GroupNorm of the retention output followed by the SiLU gate
    (Edifice.Attention.RetNet, "Multi-Scale Retention (MSR)": GroupNorm over heads, then
    Y = SiLU(X W_G) * GroupNorm(Retention(X))), fp64.  Each (batch, head, token) row of DHV
    values is one group: y = (h - mean) / sqrt(var + eps) * weight + bias with the biased
    variance, then y *= silu(g).  The projections X W_G (given here as g) and W_O are
    matrix products outside the recurrence.

    h, g: [B,NH,S,DHV] (g None = no gate); weight, bias: [NH*DHV] per channel (None = 1, 0).
    Returns y, fp64.
    """
    h = np.asarray(h, dtype=np.float64)
    B, NH, S, DHV = h.shape
    mu = h.mean(axis=-1, keepdims=True)
    var = ((h - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (h - mu) / np.sqrt(var + eps)
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float64).reshape(1, NH, 1, DHV)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64).reshape(1, NH, 1, DHV)
    if g is not None:
        y = y * silu(g)
    return y


def retention_block(q, k, v, igate=None, fgate=None, g=None, gn_weight=None, gn_bias=None,
                    C0=None, n0=None, m0=None, *, pos0=None, theta_base: float = 10000.0,
                    eps: float = 1e-5, num_blocks: int = 1, retention: bool = True, rounding=None):
    """The multi-scale retention block around the recurrence, in the page's order
    (Edifice.Attention.RetNet, "Key Innovation" and "Multi-Scale Retention (MSR)"): rotate q
    and k by Theta, run the recurrence (``sequential``), GroupNorm each head's output and
    gate it with SiLU(g).  ``rounding`` (None or a function) is applied to the rotated q, k
    and to h before the GroupNorm, to model a storage precision between the steps.

    Returns (y, C, n, m) as ``sequential`` does (n, m None in retention mode).
    """
    qr, kr = theta_rotate(q, pos0, theta_base), theta_rotate(k, pos0, theta_base)
    if rounding is not None:
        qr, kr = rounding(qr), rounding(kr)
    h, C, n, m = sequential(qr, kr, v, igate, fgate, None, C0, n0, m0, num_blocks=num_blocks,
                            retention=retention)
    if rounding is not None:
        h = rounding(h)
    return group_norm_gate(h, g, gn_weight, gn_bias, eps), C, n, m


def gdn2_sequential(q, k, v, g, b, w, S0=None):
    """Gated DeltaNet-2 (burn-gdn2 config.rs: channel-wise erase gate b in [0,1]^{d_k}, write
    gate w in [0,1]^{d_v}, state S [B,H,K,V] carried token by token), fp64, one token at a time.
    The page gives the gates' roles and the reductions (b = w = beta 1 is KDA; a scalar decay
    on top is Gated DeltaNet), not the update itself; the reading built here is the KDA step
    with its erase and write strengths split by channel:

        S'_t = Diag(alpha_t) S_{t-1}                 (alpha_t = exp(g_t), per key channel)
        r_t  = S'_t^T k_t                            (the value stored under k_t)
        S_t  = S'_t - (b_t o k_t) r_t^T + k_t (w_t o v_t)^T
        o_t  = S_t^T q_t

    q, k, g, b: [B,H,T,K] (g = log alpha <= 0); v, w: [B,H,T,V]; S0: [B,H,K,V] or None.
    Returns (o [B,H,T,V], S_T [B,H,K,V]).
    """
    q, k, v, g, b, w = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, b, w))
    B, H, T, K = q.shape
    V = v.shape[-1]
    S = np.zeros((B, H, K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((B, H, T, V))
    for t in range(T):
        Sd = np.exp(g[:, :, t])[..., None] * S
        r = np.einsum("bhkv,bhk->bhv", Sd, k[:, :, t])
        S = Sd - np.einsum("bhk,bhv->bhkv", b[:, :, t] * k[:, :, t], r) \
            + np.einsum("bhk,bhv->bhkv", k[:, :, t], w[:, :, t] * v[:, :, t])
        o[:, :, t] = np.einsum("bhkv,bhk->bhv", S, q[:, :, t])
    return o, S


def gdn2_chunk(q, k, v, g, b, w, S0=None, chunk: int = 64):
    """The chunked evaluation of ``gdn2_sequential`` (burn-gdn2 Gdn2Mode::Chunk: intra-chunk
    interactions as dense products with a WY-like triangular solve, the state carried between
    chunks), fp64, written from this derivation.  Inside a chunk with cumulative log decay
    G_t = sum_{s<=t} g_s (per key channel) and carried state S0:

        r_t = (k_t o e^{G_t})^T S0 + sum_{s<t} [sum_i k_ti k_si e^{G_ti-G_si}] u_s
                                   - sum_{s<t} [sum_i k_ti bk_si e^{G_ti-G_si}] r_s
        (u = w o v, bk = b o k), i.e. (I + L_E) R = C S0 + L_A U with strictly lower
        triangular L_A, L_E: R comes from one unit-lower-triangular solve;
        o_t = (q_t o e^{G_t})^T S0 + sum_{s<=t} [q.k weights] u_s - sum_{s<=t} [q.bk weights] r_s
        S_L = e^{G_L} o S0 + sum_s (e^{G_L - G_s} o k_s) u_s^T - sum_s (e^{G_L - G_s} o bk_s) r_s^T

    Every exponent above is <= 0.  Returns (o, S_T) like ``gdn2_sequential``.
    """
    q, k, v, g, b, w = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, b, w))
    B, H, T, K = q.shape
    V = v.shape[-1]
    S = np.zeros((B, H, K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((B, H, T, V))
    for bb in range(B):
        for hh in range(H):
            St = S[bb, hh].copy()
            for c0 in range(0, T, chunk):
                sl = slice(c0, min(T, c0 + chunk))
                qc, kc, gc = q[bb, hh, sl], k[bb, hh, sl], g[bb, hh, sl]
                u = w[bb, hh, sl] * v[bb, hh, sl]
                bk = b[bb, hh, sl] * kc
                G = np.cumsum(gc, axis=0)                        # [L, K]
                Lc = G.shape[0]
                dec = np.exp(np.minimum(G[:, None, :] - G[None, :, :], 0.0))  # [t, s, K]; s <= t used
                low = np.tril(np.ones((Lc, Lc)), -1)
                incl = np.tril(np.ones((Lc, Lc)))
                LA = np.einsum("ti,si,tsi->ts", kc, kc, np.where(low[..., None] > 0, dec, 0.0))
                LE = np.einsum("ti,si,tsi->ts", kc, bk, np.where(low[..., None] > 0, dec, 0.0))
                rhs = (kc * np.exp(G)) @ St + LA @ u
                R = np.linalg.solve(np.eye(Lc) + LE, rhs)
                QA = np.einsum("ti,si,tsi->ts", qc, kc, np.where(incl[..., None] > 0, dec, 0.0))
                QE = np.einsum("ti,si,tsi->ts", qc, bk, np.where(incl[..., None] > 0, dec, 0.0))
                o[bb, hh, sl] = (qc * np.exp(G)) @ St + QA @ u - QE @ R
                tail = np.exp(G[-1][None, :] - G)                # [L, K]
                St = np.exp(G[-1])[:, None] * St + (tail * kc).T @ u - (tail * bk).T @ R
            S[bb, hh] = St
    return o, S


def state_bytes(layers: int, heads: int, dqk: int, dv: int, bytes_per_value: int) -> int:
    """Bytes of recurrent state per sequence: per head a dv x dqk matrix, a dqk
    normaliser and one stabiliser scalar (xLSTM 7B "Modelled costs": the state
    does not grow with context)."""
    return layers * heads * (dqk * dv + dqk + 1) * bytes_per_value
