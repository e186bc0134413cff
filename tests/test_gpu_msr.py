"""GPU parity of the steps either side of retention (Edifice.Attention.RetNet, "Key Innovation"
and "Multi-Scale Retention (MSR)"): mlstm_theta_rotate, mlstm_group_norm_gate and the block
mlstm_fwd_chunkwise_msr, against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import TOL, TORCH_DTYPE, dev, host, m_err, slice_relerr

pytestmark = pytest.mark.gpu


def bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def rounding_of(dtype):
    if dtype == "bf16":
        return bf16_round
    return lambda x: np.asarray(x, dtype=np.float32).astype(np.float64)


@pytest.mark.parametrize("dtype,D,inplace", [("f32", 64, False), ("bf16", 64, True), ("bf16", 256, False),
                                             ("f32", 12, False)])
def test_theta_rotate(dtype, D, inplace):
    rng = np.random.default_rng(61)
    B, NH, S = 3, 5, 131
    td = TORCH_DTYPE[dtype]
    q = torch.from_numpy(rng.standard_normal((B, NH, S, D)).astype(np.float32)).to(td)
    k = torch.from_numpy(rng.standard_normal((B, NH, S, D)).astype(np.float32) * 0.1).to(td)
    pos0 = np.array([0, 5000, 123], dtype=np.int64)
    qh, kh = q.float().numpy(), k.float().numpy()
    qd, kd = q.cuda(), k.cuda()
    qo, ko = mlstm.theta_rotate(qd, kd, torch.from_numpy(pos0).cuda(), 10000.0,
                                q_out=qd if inplace else None, k_out=kd if inplace else None)
    torch.cuda.synchronize()
    tol = 2e-6 if dtype == "f32" else 8e-3  # fp32 products; one bf16 rounding of the output
    for got, x in ((qo, qh), (ko, kh)):
        ref = oracle.theta_rotate(x, pos0, 10000.0)
        assert slice_relerr(host(got), ref, 3) <= tol


@pytest.mark.parametrize("dtype,DHV,gate,affine", [("f32", 64, True, True), ("bf16", 64, True, False),
                                                   ("bf16", 512, True, True), ("f32", 16, False, False),
                                                   ("bf16", 2048, False, True)])
def test_group_norm_gate(dtype, DHV, gate, affine):
    rng = np.random.default_rng(62)
    B, NH, S = 2, 3, 37
    td = TORCH_DTYPE[dtype]
    h = torch.from_numpy((rng.standard_normal((B, NH, S, DHV)) * 2 + 0.5).astype(np.float32)).to(td)
    g = torch.from_numpy(rng.standard_normal((B, NH, S, DHV)).astype(np.float32)).to(td) if gate else None
    w = rng.standard_normal(NH * DHV).astype(np.float32) if affine else None
    b = rng.standard_normal(NH * DHV).astype(np.float32) if affine else None
    y = mlstm.group_norm_gate(h.cuda(), g.cuda() if gate else None, dev(w), dev(b), 1e-5)
    torch.cuda.synchronize()
    ref = oracle.group_norm_gate(h.float().numpy(), g.float().numpy() if gate else None, w, b, 1e-5)
    assert slice_relerr(host(y), ref, 3) <= TOL[dtype]
    # in place
    hd = h.cuda()
    mlstm.group_norm_gate(hd, g.cuda() if gate else None, dev(w), dev(b), 1e-5, y=hd)
    torch.cuda.synchronize()
    assert slice_relerr(host(hd), ref, 3) <= TOL[dtype]


CASES = [
    # dtype, S, DHQK, DHV, nb, retention, with_state  (tensor-core walk for bf16, SIMT for fp32)
    ("bf16", 200, 64, 64, 1, True, False),
    ("bf16", 256, 64, 128, 1, True, True),
    ("bf16", 192, 128, 128, 2, True, False),
    ("bf16", 200, 64, 64, 1, False, True),
    ("bf16", 130, 64, 256, 1, False, False),
    ("f32", 100, 32, 32, 1, True, False),
    ("f32", 70, 32, 64, 2, False, True),
]


@pytest.mark.parametrize("dtype,S,DHQK,DHV,nb,retention,with_state", CASES)
def test_msr_block(dtype, S, DHQK, DHV, nb, retention, with_state):
    B, NH = 2, 3
    chunk = 64 if dtype == "bf16" else 16
    w = inputs.Workload(2, "msr", B, NH, S, DHQK, DHV, chunk, nb, dtype, retention, 1 / np.sqrt(DHQK // nb))
    inp = inputs.forward_inputs(w, seed=63)
    rng = np.random.default_rng(64)
    td = TORCH_DTYPE[dtype]
    g = torch.from_numpy(rng.standard_normal((B, NH, S, DHV)).astype(np.float32)).to(td).float().numpy()
    gw = (1 + 0.3 * rng.standard_normal(NH * DHV)).astype(np.float32)
    gb = (0.2 * rng.standard_normal(NH * DHV)).astype(np.float32)
    pos0 = np.array([0, 777], dtype=np.int64)
    dk, dv = DHQK // nb, DHV // nb
    C0 = n0 = m0 = None
    if with_state:
        C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
        if not retention:
            n0 = (rng.standard_normal((B, NH, nb, dk)) * 0.2).astype(np.float32)
            m0 = rng.standard_normal((B, NH)).astype(np.float32)
    ig = None if retention else dev(inp["igate"])
    fg = None if retention else dev(inp["fgate"])
    y, C, n, m = mlstm.fwd_chunkwise_msr(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), ig, fg,
                                         dev(g, td), dev(gw), dev(gb), dev(C0), dev(n0), dev(m0),
                                         pos0=torch.from_numpy(pos0).cuda(), eps=1e-5, chunk=chunk, num_blocks=nb,
                                         retention=retention)
    torch.cuda.synchronize()
    yr, Cr, nr, mr = oracle.retention_block(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"], g, gw, gb,
                                            C0, n0, m0, pos0=pos0, eps=1e-5, num_blocks=nb, retention=retention,
                                            rounding=rounding_of(dtype))
    tol = TOL[dtype]
    errs = {"y": slice_relerr(host(y), yr, 2), "C": slice_relerr(host(C), Cr, 3)}
    if not retention:
        errs["n"] = slice_relerr(host(n), nr, 3)
        errs["m"] = m_err(host(m), mr)
    assert all(e <= tol for e in errs.values()), errs


def test_msr_decode_steps_match_the_block_prefill():
    """Token by token: rotate at the sequence's position, one mlstm_step, GroupNorm + gate ==
    the block's prefill at that token (retention, bf16)."""
    B, NH, S, D = 2, 2, 9, 64
    w = inputs.Workload(2, "msr", B, NH, S, D, D, 64, 1, "bf16", True, 1 / 8)
    inp = inputs.forward_inputs(w, seed=65)
    rng = np.random.default_rng(66)
    g = torch.from_numpy(rng.standard_normal((B, NH, S, D)).astype(np.float32)).to(torch.bfloat16).cuda()
    pos0 = torch.tensor([10, 0], dtype=torch.int64, device="cuda")
    q, k, v = (dev(inp[x], torch.bfloat16) for x in ("q", "k", "v"))
    y_pre, C_pre, _, _ = mlstm.fwd_chunkwise_msr(q, k, v, g=g, pos0=pos0, retention=True)
    C = torch.zeros((B, NH, 1, D, D), dtype=torch.float32, device="cuda")
    ys = []
    for t in range(S):
        qt, kt = mlstm.theta_rotate(q[:, :, t:t + 1].contiguous(), k[:, :, t:t + 1].contiguous(), pos0 + t)
        h = torch.empty((B, NH, D), dtype=torch.bfloat16, device="cuda")
        mlstm.step(qt.reshape(B, NH, D), kt.reshape(B, NH, D), v[:, :, t].contiguous(), None, None, C, None, None,
                   h=h, retention=True)
        ys.append(mlstm.group_norm_gate(h.reshape(B, NH, 1, D), g[:, :, t:t + 1].contiguous()))
    torch.cuda.synchronize()
    y_dec = torch.cat(ys, dim=2)
    assert slice_relerr(host(y_dec), host(y_pre), 2) <= TOL["bf16"]
    assert slice_relerr(host(C), host(C_pre), 3) <= TOL["bf16"]


@pytest.mark.parametrize("S,gate,affine,with_state", [
    (1000, False, False, False),  # several segments, ragged last chunk, no gate, no affine
    (64, True, True, True),       # one chunk
    (2048, True, True, False),    # the retention-block workload's length
])
def test_msr_block_retention_heads_of_64(S, gate, affine, with_state):
    """The block on 64 x 64 retention heads in bf16 (the tensor-core walk, then the GroupNorm +
    gate pass), with and without the gate and the affine GroupNorm weights, across several
    segments and a ragged last chunk; compared with the oracle's block on the same inputs."""
    B, NH, D = 2, 4, 64
    w = inputs.Workload(2, "msr_fused", B, NH, S, D, D, 64, 1, "bf16", True, 1 / np.sqrt(D))
    p = mlstm.fwd_params(B, NH, S, D, D, 64, 1, torch.bfloat16, True)
    assert mlstm.plan(p)["tensor_core"] == 1
    inp = inputs.forward_inputs(w, seed=S + 5)
    rng = np.random.default_rng(S)
    td = torch.bfloat16
    g = torch.from_numpy(rng.standard_normal((B, NH, S, D)).astype(np.float32)).to(td).float().numpy() if gate else None
    gw = (1 + 0.3 * rng.standard_normal(NH * D)).astype(np.float32) if affine else None
    gb = (0.2 * rng.standard_normal(NH * D)).astype(np.float32) if affine else None
    C0 = (rng.standard_normal((B, NH, 1, D, D)) * 0.2).astype(np.float32) if with_state else None
    pos0 = np.array([3, 1000], dtype=np.int64)
    y, C, _, _ = mlstm.fwd_chunkwise_msr(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td), None, None,
                                         dev(g, td) if gate else None, dev(gw), dev(gb), dev(C0), None, None,
                                         pos0=torch.from_numpy(pos0).cuda(), eps=1e-5, retention=True)
    torch.cuda.synchronize()
    yr, Cr, _, _ = oracle.retention_block(inp["q"], inp["k"], inp["v"], None, None, g, gw, gb, C0, None, None,
                                          pos0=pos0, eps=1e-5, retention=True, rounding=rounding_of("bf16"))
    errs = {"y": slice_relerr(host(y), yr, 2), "C": slice_relerr(host(C), Cr, 3)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
