"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Element-by-element on the same seeded inputs.  Bounds: max relative error per
(batch, head[, block]) slice <= 1e-4 for fp32 inputs, <= 2e-2 for bf16 inputs
(fp32 state in both); m within the same bound relative to max(1, |m|).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import (TOL, TORCH_DTYPE, Guarded, conditioned_excess, dev, host, m_err, readout_scale,
                           slice_relerr)

pytestmark = pytest.mark.gpu


def guarded_outputs(B, NH, S, DHQK, DHV, nb, td, retention):
    """h and the final state as views into guard-banded buffers (tests.helpers.Guarded)."""
    g = {"h": Guarded((B, NH, S, DHV), td), "C": Guarded((B, NH, nb, DHV // nb, DHQK // nb), torch.float32)}
    if not retention:
        g["n"] = Guarded((B, NH, nb, DHQK // nb), torch.float32)
        g["m"] = Guarded((B, NH), torch.float32)
    return g


def assert_guards_intact(guards, what=""):
    bad = [key for key, gd in guards.items() if not gd.intact()]
    assert not bad, f"{what}: writes outside {bad}"


def gpu_fwd(inp, dtype, chunk, nb=1, retention=False, ogate=None, C0=None, n0=None, m0=None):
    td = TORCH_DTYPE[dtype]
    q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
    ig = None if retention else dev(inp["igate"])
    fg = None if retention else dev(inp["fgate"])
    B, NH, S, DHQK = q.shape
    gd = guarded_outputs(B, NH, S, DHQK, v.shape[-1], nb, td, retention)
    out = {key: gd[key].t if key in gd else None for key in ("h", "C", "n", "m")}
    h, C, n, m = mlstm.fwd_chunkwise(q, k, v, ig, fg, dev(ogate, td) if ogate is not None else None,
                                     dev(C0), dev(n0), dev(m0), chunk=chunk, num_blocks=nb, retention=retention,
                                     h=out["h"], C_out=out["C"], n_out=out["n"], m_out=out["m"])
    torch.cuda.synchronize()
    assert_guards_intact(gd, f"S={S} chunk={chunk} nb={nb}")
    return host(h), host(C), host(n), host(m)


def oracle_fwd(inp, nb=1, retention=False, ogate=None, C0=None, n0=None, m0=None):
    if retention:
        return oracle.sequential(inp["q"], inp["k"], inp["v"], C0=C0, num_blocks=nb, retention=True)
    return oracle.sequential(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"], ogate, C0, n0, m0,
                             num_blocks=nb)


def check(got, ref, dtype, retention=False, what=""):
    tol = TOL[dtype]
    h, C, n, m = got
    hr, Cr, nr, mr = ref
    errs = {"h": slice_relerr(h, hr, 2), "C": slice_relerr(C, Cr, 3)}
    if not retention:
        errs["n"] = slice_relerr(n, nr, 3)
        errs["m"] = m_err(m, mr)
    bad = {key: val for key, val in errs.items() if not val <= tol}
    assert not bad, f"{what} errors above {tol}: {errs}"
    return errs


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_workload_forward_parity(idx):
    w = inputs.WORKLOADS[idx]
    inp = inputs.forward_inputs(w)
    got = gpu_fwd(inp, w.dtype, w.chunk, w.num_blocks, w.retention)
    ref = oracle_fwd(inp, w.num_blocks, w.retention)
    errs = check(got, ref, w.dtype, w.retention, w.describe())
    print(w.describe(), errs)


@pytest.mark.parametrize("S,chunk", [(70, 16), (1, 16), (5, 64), (16, 1), (33, 8), (128, 128)])
def test_forward_ragged_and_small(S, chunk):
    w = inputs.WORKLOADS[0]
    inp = inputs.forward_inputs(w, seed=7, S=S)
    check(gpu_fwd(inp, "f32", chunk), oracle_fwd(inp), "f32", what=f"S={S} chunk={chunk}")


def test_forward_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(3)
    C0 = rng.standard_normal((1, 2, 1, 16, 16)).astype(np.float32)
    n0 = rng.standard_normal((1, 2, 1, 16)).astype(np.float32)
    m0 = rng.standard_normal((1, 2)).astype(np.float32)
    z = np.zeros((1, 2, 0, 16), np.float32)
    inp = dict(q=z, k=z, v=z, igate=np.zeros((1, 2, 0), np.float32), fgate=np.zeros((1, 2, 0), np.float32))
    h, C, n, m = gpu_fwd(inp, "f32", 16, C0=C0, n0=n0, m0=m0)
    assert h.shape == (1, 2, 0, 16)
    assert np.array_equal(C, C0) and np.array_equal(n, n0) and np.array_equal(m, m0)


def test_forward_empty_batch():
    z = np.zeros((0, 2, 8, 16), np.float32)
    g = np.zeros((0, 2, 8), np.float32)
    h, C, n, m = gpu_fwd(dict(q=z, k=z, v=z, igate=g, fgate=g), "f32", 4)
    assert h.shape == (0, 2, 8, 16) and C.shape == (0, 2, 1, 16, 16)


@pytest.mark.parametrize("dtype,nb", [("f32", 1), ("bf16", 1), ("f32", 2), ("bf16", 4)])
def test_forward_initial_state_and_output_gate(dtype, nb):
    rng = np.random.default_rng(11)
    B, NH, S, DHQK, DHV = 2, 3, 100, 32, 64
    w = inputs.Workload(0, "t", B, NH, S, DHQK, DHV, 16, nb, dtype, False, 1 / np.sqrt(DHQK))
    inp = inputs.forward_inputs(w, seed=12)
    dk, dv = DHQK // nb, DHV // nb
    C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.3).astype(np.float32)
    n0 = (rng.standard_normal((B, NH, nb, dk)) * 0.3).astype(np.float32)
    m0 = rng.standard_normal((B, NH)).astype(np.float32)
    og = inputs.round_to(1 / (1 + np.exp(-rng.standard_normal((B, NH, S, DHV)))), dtype)
    got = gpu_fwd(inp, dtype, 16, nb, ogate=og, C0=C0, n0=n0, m0=m0)
    ref = oracle_fwd(inp, nb, ogate=og, C0=C0, n0=n0, m0=m0)
    check(got, ref, dtype, what=f"{dtype} nb={nb}")


def test_forward_state_in_place():
    w = inputs.WORKLOADS[0]
    inp = inputs.forward_inputs(w, seed=21)
    rng = np.random.default_rng(22)
    C0 = (rng.standard_normal((1, 2, 1, 16, 16)) * 0.2).astype(np.float32)
    n0 = (rng.standard_normal((1, 2, 1, 16)) * 0.2).astype(np.float32)
    m0 = rng.standard_normal((1, 2)).astype(np.float32)
    C, n, m = dev(C0), dev(n0), dev(m0)
    q, k, v, ig, fg = (dev(inp[x]) for x in ("q", "k", "v", "igate", "fgate"))
    h, C2, n2, m2 = mlstm.fwd_chunkwise(q, k, v, ig, fg, None, C, n, m, chunk=16, C_out=C, n_out=n, m_out=m)
    torch.cuda.synchronize()
    assert C2.data_ptr() == C.data_ptr()
    ref = oracle_fwd(inp, C0=C0, n0=n0, m0=m0)
    check((host(h), host(C), host(n), host(m)), ref, "f32", what="in place")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_retention_with_initial_state(dtype):
    rng = np.random.default_rng(31)
    w = inputs.Workload(2, "r", 2, 4, 90, 32, 48, 16, 1, dtype, True, 1 / np.sqrt(32))
    inp = inputs.forward_inputs(w, seed=32)
    C0 = (rng.standard_normal((2, 4, 1, 48, 32)) * 0.2).astype(np.float32)
    got = gpu_fwd(inp, dtype, 16, retention=True, C0=C0)
    ref = oracle_fwd(inp, retention=True, C0=C0)
    check(got, ref, dtype, retention=True, what="retention C0")


def test_split_prefill_resume_equals_one_prefill():
    w = inputs.Workload(1, "s", 2, 2, 192, 64, 64, 64, 2, "bf16", False, 1 / 8)
    inp = inputs.forward_inputs(w, seed=41)
    td = torch.bfloat16
    q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
    ig, fg = dev(inp["igate"]), dev(inp["fgate"])
    h, C, n, m = mlstm.fwd_chunkwise(q, k, v, ig, fg, chunk=64, num_blocks=2)
    cut = 100
    sl = lambda t: t[:, :, :cut].contiguous()
    sr = lambda t: t[:, :, cut:].contiguous()
    h1, C1, n1, m1 = mlstm.fwd_chunkwise(sl(q), sl(k), sl(v), sl(ig), sl(fg), chunk=64, num_blocks=2)
    h2, C2, n2, m2 = mlstm.fwd_chunkwise(sr(q), sr(k), sr(v), sr(ig), sr(fg), None, C1, n1, m1, chunk=64,
                                         num_blocks=2)
    torch.cuda.synchronize()
    ref = oracle_fwd(inp, 2)
    check((host(torch.cat([h1, h2], 2)), host(C2), host(n2), host(m2)), ref, "bf16", what="split")
    check((host(h), host(C), host(n), host(m)), ref, "bf16", what="one pass")


@pytest.mark.parametrize("dtype,nb,retention", [("f32", 1, False), ("bf16", 2, False), ("bf16", 1, True)])
def test_prefill_then_decode_steps_equals_longer_prefill(dtype, nb, retention):
    B, NH, S, K, DHQK, DHV = 2, 2, 80, 12, 64, 32
    w = inputs.Workload(0, "x", B, NH, S + K, DHQK, DHV, 16, nb, dtype, retention, 1 / 8)
    inp = inputs.forward_inputs(w, seed=51)
    td = TORCH_DTYPE[dtype]
    q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
    ig, fg = dev(inp["igate"]), dev(inp["fgate"])
    pre = lambda t: t[:, :, :S].contiguous()
    gi = (None, None) if retention else (pre(ig), pre(fg))
    h, C, n, m = mlstm.fwd_chunkwise(pre(q), pre(k), pre(v), *gi, chunk=16, num_blocks=nb, retention=retention)
    hs = [h]
    for t in range(S, S + K):
        g2 = (None, None) if retention else (ig[:, :, t].contiguous(), fg[:, :, t].contiguous())
        ht = mlstm.step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(), *g2, C, n, m,
                        num_blocks=nb, retention=retention)
        hs.append(ht[:, :, None])
    torch.cuda.synchronize()
    ref = oracle_fwd(inp, nb, retention)
    check((host(torch.cat(hs, 2)), host(C), host(n), host(m)), ref, dtype, retention, "prefill+steps")


@pytest.mark.parametrize("dk", [4, 8, 16, 32, 64, 128, 256, 512])
def test_decode_key_widths(dk):
    B, NH, T, dv = 3, 2, 6, 40
    w = inputs.Workload(4, "d", B, NH, T, dk, dv, 1, 1, "f32", False, 1 / np.sqrt(dk))
    inp = inputs.forward_inputs(w, seed=60 + dk)
    rng = np.random.default_rng(dk)
    C0 = (rng.standard_normal((B, NH, 1, dv, dk)) * 0.1).astype(np.float32)
    n0 = (rng.standard_normal((B, NH, 1, dk)) * 0.1).astype(np.float32)
    m0 = rng.standard_normal((B, NH)).astype(np.float32)
    C, n, m = dev(C0), dev(n0), dev(m0)
    hs = []
    for t in range(T):
        step_in = [dev(np.ascontiguousarray(inp[x][:, :, t])) for x in ("q", "k", "v", "igate", "fgate")]
        hs.append(mlstm.step(*step_in, C, n, m)[:, :, None])
    torch.cuda.synchronize()
    ref = oracle_fwd(inp, C0=C0, n0=n0, m0=m0)
    check((host(torch.cat(hs, 2)), host(C), host(n), host(m)), ref, "f32", what=f"decode dk={dk}")


@pytest.mark.parametrize("retention,og", [(True, False), (False, True)])
def test_decode_retention_and_output_gate(retention, og):
    B, NH, T, DHQK, DHV = 4, 8, 5, 64, 64
    w = inputs.Workload(4, "d", B, NH, T, DHQK, DHV, 1, 1, "bf16", retention, 1 / 8)
    inp = inputs.forward_inputs(w, seed=70)
    rng = np.random.default_rng(71)
    C0 = (rng.standard_normal((B, NH, 1, DHV, DHQK)) * 0.1).astype(np.float32)
    n0 = (rng.standard_normal((B, NH, 1, DHQK)) * 0.1).astype(np.float32)
    m0 = np.zeros((B, NH), np.float32)
    ogv = inputs.round_to(rng.uniform(0, 1, (B, NH, T, DHV)), "bf16") if og else None
    C, n, m = dev(C0), dev(n0), dev(m0)
    hs = []
    for t in range(T):
        x = [dev(np.ascontiguousarray(inp[key][:, :, t]), torch.bfloat16) for key in ("q", "k", "v")]
        g = (None, None) if retention else [dev(np.ascontiguousarray(inp[key][:, :, t])) for key in ("igate", "fgate")]
        o = dev(np.ascontiguousarray(ogv[:, :, t]), torch.bfloat16) if og else None
        hs.append(mlstm.step(*x, *g, C, None if retention else n, None if retention else m, o,
                             retention=retention)[:, :, None])
    torch.cuda.synchronize()
    if retention:
        ref = oracle.sequential(inp["q"], inp["k"], inp["v"], C0=C0, retention=True)
        got = (host(torch.cat(hs, 2)), host(C), None, None)
    else:
        ref = oracle_fwd(inp, ogate=ogv, C0=C0, n0=n0, m0=m0)
        got = (host(torch.cat(hs, 2)), host(C), host(n), host(m))
    check(got, ref, "bf16", retention, "decode")


def test_large_input_gates_stay_finite():
    # exp(60) overflows fp32 without the stabiliser.  With igate ~ 60 the floor e^{-m} of the
    # denominator is ~e^{-61}, so a random sign pattern of n.q could cancel to near zero and make
    # h ill-conditioned in any fp32 evaluation; non-negative q and k keep n.q a sum of positive
    # terms, so the test measures the stabiliser and not that conditioning.
    w = inputs.WORKLOADS[0]
    inp = inputs.forward_inputs(w, seed=80)
    inp["q"], inp["k"] = np.abs(inp["q"]), np.abs(inp["k"])
    inp["igate"] = inp["igate"] + 60.0
    got = gpu_fwd(inp, "f32", 16)
    assert all(np.all(np.isfinite(x)) for x in got)
    check(got, oracle_fwd(inp), "f32", what="large igate")


def test_large_input_gates_signed_inputs_within_conditioned_bound():
    # The same input gates with q and k of both signs.  n'.q (and C'q) can now cancel: a token
    # whose read-out terms sum to many times the read-out loses that factor of the relative
    # accuracy of those terms, in any fixed-precision evaluation (tests.helpers.readout_scale).
    # The bound per element is the fp32 tolerance relative to the token's own read-out plus
    # 2^-20 (sixteen fp32 roundings) kappa_t (h_abs + |h|).
    w = inputs.WORKLOADS[0]
    inp = inputs.forward_inputs(w, seed=80)
    inp["igate"] = inp["igate"] + 60.0
    got = gpu_fwd(inp, "f32", 16)
    assert all(np.all(np.isfinite(x)) for x in got)
    ref = oracle_fwd(inp)
    kappa, h_abs = readout_scale(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"])
    assert kappa.max() > 1e3  # the case really has cancelling denominators
    excess = conditioned_excess(got[0], ref[0], kappa, h_abs, TOL["f32"], 2.0 ** -20)
    assert excess <= 1.0, excess
    errs = {"C": slice_relerr(got[1], ref[1], 3), "n": slice_relerr(got[2], ref[2], 3), "m": m_err(got[3], ref[3])}
    assert all(e <= TOL["f32"] for e in errs.values()), errs


@pytest.fixture(scope="module")
def decode_workload():
    w = inputs.WORKLOADS[4]
    C0, n0, m0 = inputs.decode_initial_state(w)
    seq = inputs.decode_sequence_inputs(w, w.steps)
    return w, C0, n0, m0, seq


def test_decode_workload_parity(decode_workload):
    """Full decode workload: B128 NH8 256x512, 1024 in-place steps on the GPU; the oracle
    recomputes 16 sampled (batch, head) slices over all 1024 steps."""
    w, C0, n0, m0, seq = decode_workload
    T = w.steps
    td = torch.bfloat16
    stacked = {key: dev(np.ascontiguousarray(np.moveaxis(seq[key], 2, 0)), td if key in "qkv" else torch.float32)
               for key in ("q", "k", "v", "igate", "fgate")}
    C, n, m = dev(C0), dev(n0), dev(m0)
    h_all = torch.empty((T, w.B, w.NH, w.DHV), dtype=td, device="cuda")
    for t in range(T):
        mlstm.step(stacked["q"][t], stacked["k"][t], stacked["v"][t], stacked["igate"][t], stacked["fgate"][t],
                   C, n, m, h=h_all[t])
    torch.cuda.synchronize()
    rng = np.random.default_rng(99)
    picks = [(int(b), int(hd)) for b, hd in zip(rng.choice(w.B, 16), rng.choice(w.NH, 16))]
    bs = [b for b, _ in picks]
    hs = [hd for _, hd in picks]
    sub = lambda x: x[bs, hs][:, None]
    ref = oracle.sequential(sub(seq["q"]), sub(seq["k"]), sub(seq["v"]), sub(seq["igate"]), sub(seq["fgate"]),
                            None, C0[bs, hs][:, None], n0[bs, hs][:, None], m0[bs, hs][:, None])
    h = host(h_all).transpose(1, 2, 0, 3)[bs, hs][:, None]
    got = (h, host(C)[bs, hs][:, None], host(n)[bs, hs][:, None], host(m)[bs, hs][:, None])
    errs = check(got, ref, "bf16", what="decode workload")
    print("decode workload", errs)


# ---------------------------------------------------------------- tensor-core path
TC_CASES = [
    # B, NH, S, DHQK, DHV, nb, retention, with_state, with_o
    (2, 3, 1000, 128, 128, 1, False, True, True),
    (1, 2, 777, 256, 192, 1, False, True, False),
    (2, 2, 640, 128, 256, 2, False, True, True),
    (2, 4, 900, 64, 64, 1, True, True, False),
    (1, 1, 64, 64, 64, 1, False, False, False),
    (1, 2, 130, 64, 128, 1, False, True, False),
    (1, 8, 4096, 256, 512, 1, False, True, True),
    # heads of two and four value tiles
    (1, 2, 1000, 128, 256, 1, False, True, True),
    (2, 2, 700, 64, 256, 1, True, True, False),
    (1, 3, 777, 64, 512, 1, False, True, True),
    # blocks narrower than 64 (zero-padded tiles): 32 x 32, 16 x 16 over several segments,
    # 32 x 128 (keys padded), 64 x 32 (values padded)
    (2, 2, 300, 64, 64, 2, False, True, True),
    (1, 2, 1000, 64, 64, 4, False, True, True),
    (2, 2, 256, 64, 256, 2, False, False, False),
    (1, 2, 700, 128, 64, 2, True, True, False),
    (1, 3, 200, 32, 32, 2, False, True, False),
]


@pytest.mark.parametrize("case", TC_CASES, ids=[f"B{c[0]}NH{c[1]}S{c[2]}k{c[3]}v{c[4]}nb{c[5]}{'r' if c[6] else ''}"
                                                for c in TC_CASES])
def test_tensor_core_path(case):
    B, NH, S, DHQK, DHV, nb, retention, with_state, with_o = case
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, torch.bfloat16, retention)
    plan = mlstm.plan(p)
    assert plan["tensor_core"] == 1, plan
    w = inputs.Workload(3, "tc", B, NH, S, DHQK, DHV, 64, nb, "bf16", retention, 1 / np.sqrt(DHQK))
    inp = inputs.forward_inputs(w, seed=sum(case[:5]))
    rng = np.random.default_rng(7)
    dk, dv = DHQK // nb, DHV // nb
    C0 = n0 = m0 = og = None
    if with_state:
        C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
        if not retention:
            n0 = (rng.standard_normal((B, NH, nb, dk)) * 0.2).astype(np.float32)
            m0 = rng.standard_normal((B, NH)).astype(np.float32)
    if with_o:
        og = inputs.round_to(rng.uniform(0, 1, (B, NH, S, DHV)), "bf16")
    td = torch.bfloat16
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device="cuda")
    ws[:4] = 255
    gd = guarded_outputs(B, NH, S, DHQK, DHV, nb, td, retention)
    h, C, n, m = mlstm.fwd_chunkwise(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td),
                                     None if retention else dev(inp["igate"]), None if retention else dev(inp["fgate"]),
                                     dev(og, td) if og is not None else None, dev(C0), dev(n0), dev(m0),
                                     chunk=64, num_blocks=nb, retention=retention, workspace=ws,
                                     h=gd["h"].t, C_out=gd["C"].t, n_out=gd["n"].t if not retention else None,
                                     m_out=gd["m"].t if not retention else None)
    assert mlstm.fwd_status(p, ws) == 0, "a bounded wait expired in the kernel"
    assert_guards_intact(gd, f"tc {case}")
    ref = oracle_fwd(inp, nb, retention, og, C0, n0, m0)
    errs = check((host(h), host(C), host(n), host(m)), ref, "bf16", retention, f"tc {case} plan {plan}")
    print(case, plan, errs)


def test_tensor_core_state_in_place_across_segments():
    B, NH, S, DHQK, DHV = 1, 2, 2048, 128, 128
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, 1, torch.bfloat16, False)
    assert mlstm.plan(p)["segments"] > 1
    w = inputs.Workload(3, "tcip", B, NH, S, DHQK, DHV, 64, 1, "bf16", False, 1 / np.sqrt(DHQK))
    inp = inputs.forward_inputs(w, seed=5)
    rng = np.random.default_rng(9)
    C0 = (rng.standard_normal((B, NH, 1, DHV, DHQK)) * 0.2).astype(np.float32)
    n0 = (rng.standard_normal((B, NH, 1, DHQK)) * 0.2).astype(np.float32)
    m0 = rng.standard_normal((B, NH)).astype(np.float32)
    C, n, m = dev(C0), dev(n0), dev(m0)
    td = torch.bfloat16
    h, _, _, _ = mlstm.fwd_chunkwise(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), dev(inp["igate"]),
                                     dev(inp["fgate"]), None, C, n, m, chunk=64, C_out=C, n_out=n, m_out=m)
    torch.cuda.synchronize()
    ref = oracle_fwd(inp, C0=C0, n0=n0, m0=m0)
    check((host(h), host(C), host(n), host(m)), ref, "bf16", what="tc in place")


def test_tensor_core_wait_limit_reports_timeout_then_workspace_is_reusable():
    """A wait limit far shorter than a TMA load: the first wait on the loaded operands runs out,
    the kernels stop, drain their own copies and free their tensor memory, and the status call
    reports MLSTM_ERR_TIMEOUT promptly instead of hanging.  The same workspace then serves a
    normal call, which matches the oracle and reports no timeout."""
    import time
    B, NH, S, DHQK, DHV = 1, 2, 640, 128, 128
    w = inputs.Workload(3, "wait", B, NH, S, DHQK, DHV, 64, 1, "bf16", False, 1 / np.sqrt(DHQK))
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, 1, torch.bfloat16, False)
    plan = mlstm.plan(p)
    assert plan["tensor_core"] == 1 and plan["segments"] > 1  # both kernels with waits run
    inp = inputs.forward_inputs(w, seed=3)
    td = torch.bfloat16
    args = (dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), dev(inp["igate"]), dev(inp["fgate"]))
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device="cuda")
    short = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, 1, torch.bfloat16, False, wait_limit_cycles=256)
    t0 = time.perf_counter()
    mlstm.fwd_chunkwise(*args, chunk=64, workspace=ws, wait_limit_cycles=256)
    st = mlstm.fwd_status(short, ws)
    elapsed = time.perf_counter() - t0
    assert st == 8, mlstm.status_string(st)  # MLSTM_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed
    h, C, n, m = mlstm.fwd_chunkwise(*args, chunk=64, workspace=ws)
    assert mlstm.fwd_status(p, ws) == 0
    check((host(h), host(C), host(n), host(m)), oracle_fwd(inp), "bf16", what="after a timeout")


# Gate regimes for the tensor-core walk: the state is kept in a lazily scaled form and a
# chunk whose input gate rises far above the running stabiliser is evaluated in the
# per-element stabilised form.  Each regime runs twice: with q, k and n0 >= 0 (n.q a sum of
# positive terms, so the comparison isolates the stabilisation) and with q, k and n0 drawn
# with both signs as in every other test (signs of the Q scaling, the column and row factors
# and the guarded update weights all matter there).
GATE_REGIMES = {
    "spikes_80": dict(spikes=80.0),         # isolated input gates 80 above the rest
    "spikes_40": dict(spikes=40.0),         # large but within the lazily scaled range
    "shift_60": dict(shift=60.0),           # every input gate 60 above the initial stabiliser
    "steep_forget": dict(fmean=-1.0),       # log f ~ -1.3 per token: ~-80 per chunk
    "flat_forget": dict(fmean=8.0),         # f ~ 1: the scale barely moves
    "negative_input": dict(shift=-30.0),    # input gates far below the carried state
}


@pytest.mark.parametrize("signs", ["nonneg", "signed"])
@pytest.mark.parametrize("DHV", [128, 512])
@pytest.mark.parametrize("regime", list(GATE_REGIMES))
def test_tensor_core_gate_regimes(regime, DHV, signs):
    cfg = GATE_REGIMES[regime]
    B, NH, S, DHQK = 1, 2, 1536, 128
    w = inputs.Workload(3, "regime", B, NH, S, DHQK, DHV, 64, 1, "bf16", False, 1 / np.sqrt(DHQK))
    assert mlstm.plan(mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, 1, torch.bfloat16, False))["tensor_core"] == 1
    inp = inputs.forward_inputs(w, seed=31)
    if signs == "nonneg":
        inp["q"], inp["k"] = np.abs(inp["q"]), np.abs(inp["k"])
    rng = np.random.default_rng(32)
    if "spikes" in cfg:
        idx = rng.choice(S, size=12, replace=False)
        inp["igate"][:, :, idx] += cfg["spikes"]
    if "shift" in cfg:
        inp["igate"] = inp["igate"] + cfg["shift"]
    if "fmean" in cfg:
        inp["fgate"] = inp["fgate"] - 3.0 + cfg["fmean"]
    rs = np.random.default_rng(33)
    C0 = (rs.standard_normal((B, NH, 1, DHV, DHQK)) * 0.2).astype(np.float32)
    n0 = (rs.standard_normal((B, NH, 1, DHQK)) * 0.2).astype(np.float32)
    if signs == "nonneg":
        n0 = np.abs(n0)
    m0 = rs.standard_normal((B, NH)).astype(np.float32)
    got = gpu_fwd(inp, "bf16", 64, C0=C0, n0=n0, m0=m0)
    assert all(np.all(np.isfinite(x)) for x in got), regime
    ref = oracle_fwd(inp, C0=C0, n0=n0, m0=m0)
    if signs == "nonneg":
        print(regime, signs, check(got, ref, "bf16", what=f"{regime} {signs}"))
        return
    # Signed inputs: the final state (no cancellation) at the flat bound; h per element at the flat
    # bound relative to its own token plus 2^-8 kappa_t (h_abs + |h|) (tests.helpers.readout_scale),
    # 2^-8 being two bf16
    # roundings of the terms: the read-out reads a bf16 copy of the state, and the state itself
    # accumulates bf16 products V o u.  An input spike makes the state one dominant rank-1 term,
    # and a token whose query is nearly orthogonal to that key cancels it in num and den alike;
    # an fp64 evaluation that rounds only the read-out's copy of the state to bf16 already misses
    # the flat bound by 3x on the spike regimes (6.5 % at DHV 128, 20 % at 512).  Most tokens'
    # kappa is small, so the bound stays the flat one for them (an h of the wrong sign on one
    # token in twenty exceeds it 28-47 times in the spike and shift regimes).
    errs = {"C": slice_relerr(got[1], ref[1], 3), "n": slice_relerr(got[2], ref[2], 3), "m": m_err(got[3], ref[3])}
    assert all(e <= TOL["bf16"] for e in errs.values()), (regime, errs)
    kappa, h_abs = readout_scale(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"], C0, n0, m0)
    excess = conditioned_excess(got[0], ref[0], kappa, h_abs, TOL["bf16"], 2.0 ** -8)
    assert excess <= 1.0, (regime, excess, slice_relerr(got[0], ref[0], 2))
    print(regime, signs, errs, "h excess", excess, "flat h error", slice_relerr(got[0], ref[0], 2))


@pytest.mark.parametrize("dtype,chunk,nb,retention,with_o", [
    ("bf16", 64, 1, False, True),    # tensor-core path
    ("bf16", 64, 1, True, False),    # tensor-core path, retention
    ("f32", 16, 2, False, False),    # SIMT path, block-diagonal
])
def test_reversed_sequence_pass(dtype, chunk, nb, retention, with_o):
    """mlstm_fwd_chunkwise_reversed == the oracle on the sequence read backwards, with h put
    back at the original positions and the final state after token 0."""
    B, NH, S, DHQK, DHV = 2, 2, 333, 64, 128
    w = inputs.Workload(3, "rev", B, NH, S, DHQK, DHV, chunk, nb, dtype, retention, 1 / np.sqrt(DHQK // nb))
    inp = inputs.forward_inputs(w, seed=41)
    rng = np.random.default_rng(8)
    dk, dv = DHQK // nb, DHV // nb
    C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
    n0 = None if retention else (rng.standard_normal((B, NH, nb, dk)) * 0.2).astype(np.float32)
    m0 = None if retention else rng.standard_normal((B, NH)).astype(np.float32)
    og = None
    if with_o:
        og = (1 / (1 + np.exp(-rng.standard_normal((B, NH, S, DHV))))).astype(np.float32)
        og = torch.from_numpy(og).to(TORCH_DTYPE[dtype]).float().numpy()
    td = TORCH_DTYPE[dtype]
    q, k, v = (dev(inp[x], td) for x in ("q", "k", "v"))
    ig = None if retention else dev(inp["igate"])
    fg = None if retention else dev(inp["fgate"])
    h, C, n, m = mlstm.fwd_chunkwise(q, k, v, ig, fg, dev(og, td) if og is not None else None, dev(C0), dev(n0),
                                     dev(m0), chunk=chunk, num_blocks=nb, retention=retention, reverse=True)
    torch.cuda.synchronize()
    flip = lambda x: None if x is None else np.ascontiguousarray(np.flip(x, axis=2))
    ref = oracle_fwd({"q": flip(inp["q"]), "k": flip(inp["k"]), "v": flip(inp["v"]),
                      "igate": flip(inp.get("igate")), "fgate": flip(inp.get("fgate"))},
                     nb, retention, flip(og), C0, n0, m0)
    ref = (flip(ref[0]),) + tuple(ref[1:])
    check((host(h), host(C), host(n), host(m)), ref, dtype, retention, what="reversed")


@pytest.mark.parametrize("dtype,chunk,nb,with_o,with_state", [
    ("f32", 16, 1, False, True),
    ("bf16", 64, 2, True, True),
    ("bf16", 32, 1, False, False),
])
def test_scalar_normaliser_prefill(dtype, chunk, nb, with_o, with_state):
    """mlstm_fwd_chunkwise_scalar_normaliser == oracle.sequential_scalar_normaliser (scalar
    n_t = f n + i, denominator max(|n + bias|, 1)), h and final state."""
    B, NH, S, DHQK, DHV = 2, 3, 301, 64, 64
    w = inputs.Workload(1, "sn", B, NH, S, DHQK, DHV, chunk, nb, dtype, False, 1 / np.sqrt(DHQK // nb))
    inp = inputs.forward_inputs(w, seed=51)
    rng = np.random.default_rng(9)
    dk, dv = DHQK // nb, DHV // nb
    bias = rng.standard_normal(NH).astype(np.float32) * 2.0
    C0 = n0 = m0 = og = None
    if with_state:
        C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
        n0 = (rng.standard_normal((B, NH)) * 0.5).astype(np.float32)
        m0 = rng.standard_normal((B, NH)).astype(np.float32)
    if with_o:
        og = (1 / (1 + np.exp(-rng.standard_normal((B, NH, S, DHV))))).astype(np.float32)
        og = torch.from_numpy(og).to(TORCH_DTYPE[dtype]).float().numpy()
    td = TORCH_DTYPE[dtype]
    h, C, n, m = mlstm.fwd_chunkwise_scalar_normaliser(
        dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), dev(inp["igate"]), dev(inp["fgate"]), dev(bias),
        dev(og, td) if og is not None else None, dev(C0), dev(n0), dev(m0), chunk=chunk, num_blocks=nb)
    torch.cuda.synchronize()
    hr, Cr, nr, mr = oracle.sequential_scalar_normaliser(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"],
                                                         bias, og, C0, n0, m0, num_blocks=nb)
    tol = TOL[dtype]
    errs = {"h": slice_relerr(host(h), hr, 2), "C": slice_relerr(host(C), Cr, 3),
            "n": float(np.max(np.abs(host(n) - nr)) / max(np.max(np.abs(nr)), 1e-30)), "m": m_err(host(m), mr)}
    assert all(e <= tol for e in errs.values()), errs


SN_TC_CASES = [
    # B, NH, S, DHQK, DHV, nb, with_o, with_state
    (1, 2, 700, 128, 256, 1, True, True),      # several segments (segment summaries of the scalar n)
    (2, 2, 333, 64, 128, 1, False, False),     # ragged last chunk, zero initial state
    (1, 4, 2048, 256, 512, 1, False, True),    # the large-head shape
    (2, 2, 640, 128, 128, 2, True, True),      # two blocks sharing the head's scalar n
    (1, 2, 700, 64, 64, 2, True, True),        # 32 x 32 blocks (zero-padded tiles)
]


@pytest.mark.parametrize("case", SN_TC_CASES, ids=[f"B{c[0]}NH{c[1]}S{c[2]}k{c[3]}v{c[4]}nb{c[5]}" for c in SN_TC_CASES])
def test_scalar_normaliser_prefill_tensor_core(case):
    """The scalar-normaliser variant on the tensor-core kernels (bf16, chunk 64) against
    oracle.sequential_scalar_normaliser: h, C, the per-head n and m, outputs guard-banded."""
    B, NH, S, DHQK, DHV, nb, with_o, with_state = case
    assert mlstm.plan(mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, torch.bfloat16, False))["tensor_core"] == 1
    w = inputs.Workload(3, "sn_tc", B, NH, S, DHQK, DHV, 64, nb, "bf16", False, 1 / np.sqrt(DHQK // nb))
    inp = inputs.forward_inputs(w, seed=sum(case[:5]))
    rng = np.random.default_rng(19)
    dk, dv = DHQK // nb, DHV // nb
    bias = (rng.standard_normal(NH) * 2.0).astype(np.float32)
    C0 = n0 = m0 = og = None
    if with_state:
        C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
        n0 = (rng.standard_normal((B, NH)) * 0.5).astype(np.float32)
        m0 = rng.standard_normal((B, NH)).astype(np.float32)
    if with_o:
        og = inputs.round_to(rng.uniform(0, 1, (B, NH, S, DHV)), "bf16")
    td = torch.bfloat16
    gd = {"h": Guarded((B, NH, S, DHV), td), "C": Guarded((B, NH, nb, dv, dk), torch.float32),
          "n": Guarded((B, NH), torch.float32), "m": Guarded((B, NH), torch.float32)}
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, td, False)
    ws = torch.empty(mlstm.scalar_normaliser_workspace_size(p), dtype=torch.uint8, device="cuda")
    lib = mlstm.lib()
    ptr = lambda t: None if t is None else t.data_ptr()
    args = [dev(inp[x], td) for x in ("q", "k", "v")] + [dev(inp["igate"]), dev(inp["fgate"]),
                                                          dev(og, td) if og is not None else None, dev(bias),
                                                          dev(C0), dev(n0), dev(m0)]
    import ctypes
    st = lib.mlstm_fwd_chunkwise_scalar_normaliser(
        ctypes.byref(p), *[ptr(a) for a in args], gd["h"].t.data_ptr(), gd["C"].t.data_ptr(), gd["n"].t.data_ptr(),
        gd["m"].t.data_ptr(), ws.data_ptr(), ctypes.c_size_t(ws.numel()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, mlstm.status_string(st)
    assert mlstm.fwd_status(p, ws) == 0  # synchronises; no bounded wait ran out
    assert_guards_intact(gd, f"scalar normaliser {case}")
    hr, Cr, nr, mr = oracle.sequential_scalar_normaliser(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"],
                                                         bias, og, C0, n0, m0, num_blocks=nb)
    tol = TOL["bf16"]
    errs = {"h": slice_relerr(host(gd["h"].t), hr, 2), "C": slice_relerr(host(gd["C"].t), Cr, 3),
            "n": float(np.max(np.abs(host(gd["n"].t) - nr)) / max(np.max(np.abs(nr)), 1e-30)),
            "m": m_err(host(gd["m"].t), mr)}
    assert all(e <= tol for e in errs.values()), errs


@pytest.mark.parametrize("retention,with_o,S", [(False, True, 1500), (True, False, 1000), (False, False, 2048)])
def test_reversed_sequence_pass_several_segments(retention, with_o, S):
    """The tensor-core reversed pass reads the chunks and their rows backwards in place; with
    several sequence segments the segment summaries run backwards too.  Against the oracle on
    the flipped sequence, outputs guard-banded."""
    B, NH, DHQK, DHV = 1, 2, 128, 256
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, 1, torch.bfloat16, retention)
    plan = mlstm.plan(p)
    assert plan["tensor_core"] == 1 and plan["segments"] > 1, plan
    assert mlstm.reversed_workspace_size(p) == mlstm.workspace_size(p)  # no copies on this path
    w = inputs.Workload(3, "rev_seg", B, NH, S, DHQK, DHV, 64, 1, "bf16", retention, 1 / np.sqrt(DHQK))
    inp = inputs.forward_inputs(w, seed=S)
    rng = np.random.default_rng(S + 1)
    C0 = (rng.standard_normal((B, NH, 1, DHV, DHQK)) * 0.2).astype(np.float32)
    n0 = None if retention else (rng.standard_normal((B, NH, 1, DHQK)) * 0.2).astype(np.float32)
    m0 = None if retention else rng.standard_normal((B, NH)).astype(np.float32)
    og = inputs.round_to(rng.uniform(0, 1, (B, NH, S, DHV)), "bf16") if with_o else None
    td = torch.bfloat16
    gd = guarded_outputs(B, NH, S, DHQK, DHV, 1, td, retention)
    ws = torch.empty(mlstm.reversed_workspace_size(p), dtype=torch.uint8, device="cuda")
    h, C, n, m = mlstm.fwd_chunkwise(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td),
                                     None if retention else dev(inp["igate"]), None if retention else dev(inp["fgate"]),
                                     dev(og, td) if og is not None else None, dev(C0), dev(n0), dev(m0), chunk=64,
                                     retention=retention, reverse=True, workspace=ws, h=gd["h"].t, C_out=gd["C"].t,
                                     n_out=None if retention else gd["n"].t, m_out=None if retention else gd["m"].t)
    assert mlstm.fwd_status(p, ws) == 0
    assert_guards_intact(gd, "reversed")
    flip = lambda x: None if x is None else np.ascontiguousarray(np.flip(x, axis=2))
    ref = oracle_fwd({"q": flip(inp["q"]), "k": flip(inp["k"]), "v": flip(inp["v"]),
                      "igate": flip(inp.get("igate")), "fgate": flip(inp.get("fgate"))},
                     1, retention, flip(og), C0, n0, m0)
    ref = (flip(ref[0]),) + tuple(ref[1:])
    check((host(h), host(C), host(n), host(m)), ref, "bf16", retention, what=f"reversed S={S}")
