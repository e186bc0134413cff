"""GPU parity of Gated DeltaNet-2 (mlstm_gdn2_fwd, burn-gdn2 Gdn2Mode::FusedRecurrent and
Gdn2Mode::Chunk) against the fp64 token-by-token oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import TOL, TORCH_DTYPE, dev, host, slice_relerr

pytestmark = pytest.mark.gpu


def run(inp, dtype, mode, chunk=64, inplace=False):
    td = TORCH_DTYPE[dtype]
    S0 = dev(inp["S0"])
    o, S = mlstm.gdn2_fwd(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), dev(inp["g"]), dev(inp["b"]),
                          dev(inp["w"]), S0, mode=mode, chunk=chunk, S_out=S0 if inplace and S0 is not None else None)
    torch.cuda.synchronize()
    return host(o), host(S)


def check(inp, dtype, o, S):
    o_ref, S_ref = oracle.gdn2_sequential(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], inp["w"], inp["S0"])
    errs = {"o": slice_relerr(o, o_ref, 2), "S": slice_relerr(S, S_ref, 2)}
    assert all(e <= TOL[dtype] for e in errs.values()), errs


@pytest.mark.parametrize("dtype,T,K,V,state,inplace", [
    ("f32", 37, 64, 48, True, False), ("f32", 20, 32, 20, False, False), ("bf16", 100, 128, 128, True, True),
    ("bf16", 50, 256, 64, True, False),
])
def test_recurrent(dtype, T, K, V, state, inplace):
    inp = inputs.gdn2_inputs(2, 3, T, K, V, dtype, seed=71, with_state=state)
    o, S = run(inp, dtype, "recurrent", inplace=inplace)
    check(inp, dtype, o, S)


@pytest.mark.parametrize("dtype,T,K,V,chunk,state", [
    ("f32", 70, 64, 64, 16, True), ("f32", 33, 32, 40, 8, False), ("bf16", 130, 128, 128, 64, True),
    ("bf16", 96, 128, 128, 32, True), ("bf16", 64, 256, 64, 16, True),
])
def test_chunk(dtype, T, K, V, chunk, state):
    inp = inputs.gdn2_inputs(2, 3, T, K, V, dtype, seed=72, with_state=state)
    o, S = run(inp, dtype, "chunk", chunk=chunk)
    check(inp, dtype, o, S)


def test_chunk_strong_decay():
    """log decays down to about -20 per token: every exponent of the chunk form stays <= 0."""
    inp = inputs.gdn2_inputs(1, 2, 80, 64, 64, "f32", seed=73)
    inp["g"] = (inp["g"] * 60).astype(np.float32)
    o, S = run(inp, "f32", "chunk", chunk=32)
    check(inp, "f32", o, S)


def test_decode_steps_match_the_prefill():
    """T single-token calls with the state in place == one call over the T tokens."""
    B, H, T, K, V = 4, 2, 12, 128, 128
    inp = inputs.gdn2_inputs(B, H, T, K, V, "bf16", seed=74)
    o_ref, S_ref = run(inp, "bf16", "recurrent")
    td = torch.bfloat16
    S = dev(inp["S0"])
    outs = []
    for t in range(T):
        sl = (slice(None), slice(None), slice(t, t + 1))
        o, _ = mlstm.gdn2_fwd(dev(inp["q"][sl], td), dev(inp["k"][sl], td), dev(inp["v"][sl], td), dev(inp["g"][sl]),
                              dev(inp["b"][sl]), dev(inp["w"][sl]), S, S_out=S)
        outs.append(o)
    torch.cuda.synchronize()
    # the single-token calls run the decode kernel (another reduction order): o within one
    # bf16 rounding, the fp32 state within fp32 rounding; both against the oracle as well
    assert slice_relerr(host(torch.cat(outs, dim=2)), o_ref, 2) <= 1e-2
    assert slice_relerr(host(S), S_ref, 2) <= 1e-5
    check(inp, "bf16", host(torch.cat(outs, dim=2)), host(S))


@pytest.mark.parametrize("dtype,K,V,state", [("f32", 64, 40, True), ("bf16", 256, 96, False), ("f32", 32, 32, True),
                                             ("bf16", 128, 256, True), ("f32", 64, 128, False)])
def test_decode_step(dtype, K, V, state):
    """One token per sequence (the decode kernels: 16-byte state accesses when V is a multiple
    of 128 and K at most 128, else one column per lane), state in place, ragged value tile."""
    inp = inputs.gdn2_inputs(5, 3, 1, K, V, dtype, seed=76, with_state=state)
    o, S = run(inp, dtype, "recurrent", inplace=state)
    check(inp, dtype, o, S)


def test_empty_sequence_copies_the_state():
    inp = inputs.gdn2_inputs(2, 2, 0, 64, 64, "f32", seed=75)
    o, S = run(inp, "f32", "recurrent")
    assert o.shape == (2, 2, 0, 64)
    np.testing.assert_array_equal(S, inp["S0"])


# The chunk mode on the tensor cores (bf16, chunk 64, K = 128, V = 64 or 128): the per-chunk
# matrices built for all chunks at once, then one pass per head with the state in tensor memory.
@pytest.mark.parametrize("B,H,T,V,state,inplace", [
    (2, 3, 200, 128, True, False),   # ragged last chunk
    (1, 4, 64, 64, True, True),      # one chunk, V = 64, state in place
    (2, 2, 1, 128, False, False),    # a single token
    (1, 2, 700, 64, True, False),    # eleven chunks, V = 64
    (3, 2, 1000, 128, True, True),   # sixteen chunks, in place
    (2, 80, 130, 128, True, False),  # 480 chunk CTAs (several waves: each prefetches a later CTA's
                                     # inputs into L2), ragged last chunks of two tokens
])
def test_chunk_tensor_core(B, H, T, V, state, inplace):
    inp = inputs.gdn2_inputs(B, H, T, 128, V, "bf16", seed=80 + T, with_state=state)
    td = torch.bfloat16
    p = mlstm.gdn2_params(dev(inp["q"], td), dev(inp["v"], td), "chunk", 64)
    ws_bytes = mlstm.gdn2_workspace_size(p)
    nch = (T + 63) // 64
    assert ws_bytes == 256 + B * H * nch * (65536 + 384 * V + 512)  # the tensor-core slots
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    q = dev(inp["q"], td)
    S0 = dev(inp["S0"])
    o, S = mlstm.gdn2_fwd(q, dev(inp["k"], td), dev(inp["v"], td), dev(inp["g"]), dev(inp["b"]), dev(inp["w"]), S0,
                          mode="chunk", chunk=64, workspace=ws, S_out=S0 if inplace and S0 is not None else None)
    assert mlstm.gdn2_status(q, o, ws) == 0, "a bounded wait ran out"
    check(inp, "bf16", host(o), host(S))


def test_chunk_tensor_core_strong_decay():
    """log decays down to about -20 per token: the diagonal 16-token blocks whose decay spans
    more than e^{40} are summed pair by pair; the off-diagonal factors underflow to zero."""
    inp = inputs.gdn2_inputs(1, 2, 150, 128, 128, "bf16", seed=83)
    inp["g"] = (inp["g"] * 60).astype(np.float32)
    o, S = run(inp, "bf16", "chunk", chunk=64)
    check(inp, "bf16", o, S)


def test_chunk_tensor_core_prefill_workload_sampled():
    """The GDN-2 prefill workload (B8 H16 T2048 128 x 128, bf16) in one call; the oracle on the
    heads of the first batch entry."""
    wl = [w for w in inputs.GDN2_WORKLOADS if w.name == "gdn2_prefill"][0]
    inp = inputs.gdn2_inputs(wl.B, wl.H, wl.T, wl.K, wl.V, wl.dtype, seed=7)
    o, S = run(inp, "bf16", "chunk", chunk=64)
    sub = {k_: (None if x is None else x[:1]) for k_, x in inp.items()}
    o_ref, S_ref = oracle.gdn2_sequential(sub["q"], sub["k"], sub["v"], sub["g"], sub["b"], sub["w"], sub["S0"])
    errs = {"o": slice_relerr(o[:1], o_ref, 2), "S": slice_relerr(S[:1], S_ref, 2)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    assert np.isfinite(o).all() and np.isfinite(S).all()


def test_chunk_tensor_core_wait_limit_reports_timeout_then_workspace_is_reusable():
    """A wait bound of 256 SM cycles (shorter than any copy): the scan's first wait runs out, the
    kernel drains its copies and returns, the status call reports MLSTM_ERR_TIMEOUT promptly, and
    a normal call on the same workspace then matches the oracle."""
    import time
    inp = inputs.gdn2_inputs(1, 2, 300, 128, 128, "bf16", seed=88)
    td = torch.bfloat16
    q, k, v = dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td)
    g, b, w, S0 = dev(inp["g"]), dev(inp["b"]), dev(inp["w"]), dev(inp["S0"])
    ws = torch.empty(mlstm.gdn2_workspace_size(mlstm.gdn2_params(q, v, "chunk", 64)), dtype=torch.uint8,
                     device="cuda")
    t0 = time.time()
    mlstm.gdn2_fwd(q, k, v, g, b, w, S0, mode="chunk", chunk=64, workspace=ws, wait_limit_cycles=256)
    assert mlstm.gdn2_status(q, v, ws) == 8
    assert time.time() - t0 < 5.0
    o, S = mlstm.gdn2_fwd(q, k, v, g, b, w, S0, mode="chunk", chunk=64, workspace=ws)
    assert mlstm.gdn2_status(q, v, ws) == 0
    check(inp, "bf16", host(o), host(S))
