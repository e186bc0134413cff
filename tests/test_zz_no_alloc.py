"""The prefill entry point that allocates nothing (mlstm_fwd_chunkwise_noalloc).

It exists for callers that cannot call cudaMalloc (a host framework that owns all
device memory, or code where an allocation's implicit synchronisation is not
acceptable): instead of a caller workspace it uses one scratch buffer compiled
into the library.  These tests call it through the C ABI and compare it with the
ordinary entry point, which uses a caller-allocated workspace.  The file is named
to be collected last, so that a failure here does not hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import TOL, TORCH_DTYPE, dev, host, m_err, slice_relerr

SCRATCH = 32 << 20


def test_scratch_size_is_reported():
    assert mlstm.lib().mlstm_noalloc_scratch_bytes() == SCRATCH


def test_problem_larger_than_the_buffer_is_rejected_before_any_device_work():
    # 8 heads x 2^23 tokens of fp32 stabiliser scratch is 256 MiB > 32 MiB
    p = mlstm.fwd_params(1, 8, 1 << 23, 16, 16, 16, 1, torch.float32, False)
    assert mlstm.workspace_size(p) > SCRATCH
    fake = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(14)]
    st = mlstm.lib().mlstm_fwd_chunkwise_noalloc(ctypes.byref(p), *fake[:13], ctypes.c_void_p(0))
    assert st == 5  # MLSTM_ERR_WORKSPACE


CASES = [
    # workload index, override of S (None = full size)
    (3, None),   # large-head bf16 prefill, tensor-core path, 4 sequence segments
    (2, 512),    # retention, tensor-core path
    (0, None),   # tiny fp32, SIMT path
]


@pytest.mark.gpu
@pytest.mark.parametrize("idx,S", CASES)
def test_noalloc_matches_workspace_entry_point_on_two_calls(idx, S):
    w = inputs.WORKLOADS[idx]
    td = TORCH_DTYPE[w.dtype]
    tol = TOL[w.dtype]
    p = mlstm.fwd_params(w.B, w.NH, w.S if S is None else S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    assert mlstm.workspace_size(p) <= SCRATCH
    for call, seed in enumerate((11, 12)):  # two calls in a row, different inputs
        inp = inputs.forward_inputs(w, seed=seed, S=S)
        q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
        ig = None if w.retention else dev(inp["igate"])
        fg = None if w.retention else dev(inp["fgate"])
        kw = dict(chunk=w.chunk, num_blocks=w.num_blocks, retention=w.retention)
        ref = mlstm.fwd_chunkwise(q, k, v, ig, fg, **kw)
        got = mlstm.fwd_chunkwise_noalloc(q, k, v, ig, fg, **kw)
        torch.cuda.synchronize()
        errs = {"h": slice_relerr(host(got[0]), host(ref[0]), 2), "C": slice_relerr(host(got[1]), host(ref[1]), 3)}
        if not w.retention:
            errs["n"] = slice_relerr(host(got[2]), host(ref[2]), 3)
            errs["m"] = m_err(host(got[3]), host(ref[3]))
        assert all(e <= tol for e in errs.values()), (call, errs)
        # no bounded wait of the built-in buffer's call ran out
        assert mlstm.fwd_status(p, noalloc=True) == 0


@pytest.mark.gpu
def test_noalloc_large_head_matches_the_oracle():
    """One call on the full large-head workload (tensor-core path, 4 segments) against the fp64
    oracle directly, so that the entry point is checked on its own and not only against the
    workspace entry point."""
    w = inputs.WORKLOADS[3]
    td = TORCH_DTYPE[w.dtype]
    inp = inputs.forward_inputs(w)
    q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
    h, C, n, m = mlstm.fwd_chunkwise_noalloc(q, k, v, dev(inp["igate"]), dev(inp["fgate"]), chunk=w.chunk)
    p = mlstm.fwd_params(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.num_blocks, td, w.retention)
    assert mlstm.fwd_status(p, noalloc=True) == 0  # synchronises
    hr, Cr, nr, mr = oracle.sequential(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"])
    errs = {"h": slice_relerr(host(h), hr, 2), "C": slice_relerr(host(C), Cr, 3), "n": slice_relerr(host(n), nr, 3),
            "m": m_err(host(m), mr)}
    assert all(e <= TOL[w.dtype] for e in errs.values()), errs
