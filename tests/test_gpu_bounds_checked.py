"""The tensor-core prefill run through libmlstm_checked.so, the bounds-checked debug build: every
plain global access of its kernels checked against its buffer, every TMA coordinate against the
copy rules and every staging-tile offset against the tile, a failure recorded instead of made.
The cases cover what those checks guard: ragged tails (h rows past S stored through TMA),
several segments (summary tiles loaded back by TMA), reversed chunks, an output gate, block
slices, the scalar normaliser and retention.  Each must finish with status OK and no recorded
failure, and match the oracle as the normal build does; outputs sit between guard bands."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import TOL, Guarded, dev, host, m_err, slice_relerr
from tests.test_gpu_parity import assert_guards_intact, check, guarded_outputs, oracle_fwd

pytestmark = pytest.mark.gpu

# B, NH, S, DHQK, DHV, nb, retention, with_state, with_o, reverse
CASES = [
    (1, 2, 200, 128, 128, 1, False, True, True, False),     # one segment, ragged tail, ogate, state
    (1, 2, 1500, 128, 256, 1, False, True, False, False),   # several segments and summary units
    (2, 2, 640, 256, 512, 2, False, False, True, False),    # block slices of 128 x 256
    (1, 3, 1000, 64, 64, 1, True, True, False, False),      # retention
    (1, 2, 1500, 128, 256, 1, False, True, True, True),     # reversed, several segments, ragged
    (1, 8, 4100, 256, 512, 1, False, False, False, False),  # the large head, several segments, ragged
    (2, 2, 700, 64, 64, 2, False, True, True, False),       # 32 x 32 blocks, zero-padded tiles
    (1, 2, 600, 64, 64, 4, False, True, True, True),        # 16 x 16 blocks, reversed
]


def _ids(c):
    return f"B{c[0]}NH{c[1]}S{c[2]}k{c[3]}v{c[4]}nb{c[5]}{'r' if c[6] else ''}{'-rev' if c[9] else ''}"


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_checked_build_forward_finds_no_bad_access(case):
    B, NH, S, DHQK, DHV, nb, retention, with_state, with_o, reverse = case
    td = torch.bfloat16
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, td, retention)
    assert mlstm.plan(p)["tensor_core"] == 1
    w = inputs.Workload(3, "chk", B, NH, S, DHQK, DHV, 64, nb, "bf16", retention, 1 / np.sqrt(DHQK // nb))
    inp = inputs.forward_inputs(w, seed=S + DHV)
    rng = np.random.default_rng(S)
    dk, dv = DHQK // nb, DHV // nb
    C0 = n0 = m0 = og = None
    if with_state:
        C0 = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.2).astype(np.float32)
        if not retention:
            n0 = (rng.standard_normal((B, NH, nb, dk)) * 0.2).astype(np.float32)
            m0 = rng.standard_normal((B, NH)).astype(np.float32)
    if with_o:
        og = inputs.round_to(rng.uniform(0, 1, (B, NH, S, DHV)), "bf16")
    gd = guarded_outputs(B, NH, S, DHQK, DHV, nb, td, retention)
    with mlstm.bounds_checked() as lib:
        assert lib.mlstm_bounds_checked() == 1
        ws = torch.empty(mlstm.workspace_size(p), dtype=torch.uint8, device="cuda")
        h, C, n, m = mlstm.fwd_chunkwise(dev(inp["q"], td), dev(inp["k"], td), dev(inp["v"], td),
                                         None if retention else dev(inp["igate"]),
                                         None if retention else dev(inp["fgate"]),
                                         dev(og, td) if og is not None else None, dev(C0), dev(n0), dev(m0),
                                         chunk=64, num_blocks=nb, retention=retention, reverse=reverse,
                                         workspace=ws, h=gd["h"].t, C_out=gd["C"].t,
                                         n_out=None if retention else gd["n"].t,
                                         m_out=None if retention else gd["m"].t)
        st = mlstm.fwd_status(p, ws)
        rec = mlstm.bounds_record(p, ws)
    assert st == 0 and rec == (0, 0, 0), (mlstm.status_string(st), rec)
    assert_guards_intact(gd, f"checked {case}")
    if reverse:
        flip = lambda x: None if x is None else np.ascontiguousarray(np.flip(x, axis=2))
        ref = oracle_fwd({"q": flip(inp["q"]), "k": flip(inp["k"]), "v": flip(inp["v"]),
                          "igate": flip(inp.get("igate")), "fgate": flip(inp.get("fgate"))},
                         nb, retention, flip(og), C0, n0, m0)
        ref = (flip(ref[0]),) + tuple(ref[1:])
    elif B * NH * S * DHV > 4_000_000:  # the large head: the oracle on two heads
        sl = lambda x, a=1: None if x is None else np.ascontiguousarray(x[:, :2])
        ref = oracle_fwd({"q": sl(inp["q"]), "k": sl(inp["k"]), "v": sl(inp["v"]),
                          "igate": sl(inp.get("igate")), "fgate": sl(inp.get("fgate"))},
                         nb, retention, sl(og), sl(C0), sl(n0), sl(m0))
        check((host(h)[:, :2], host(C)[:, :2], host(n)[:, :2], host(m)[:, :2]), ref, "bf16", retention,
              what=f"checked {case}")
        return
    else:
        ref = oracle_fwd(inp, nb, retention, og, C0, n0, m0)
    check((host(h), host(C), host(n), host(m)), ref, "bf16", retention, what=f"checked {case}")


def test_checked_build_scalar_normaliser_finds_no_bad_access():
    B, NH, S, DHQK, DHV, nb = 1, 2, 1300, 128, 256, 1
    td = torch.bfloat16
    w = inputs.Workload(3, "chk_sn", B, NH, S, DHQK, DHV, 64, nb, "bf16", False, 1 / np.sqrt(DHQK))
    inp = inputs.forward_inputs(w, seed=23)
    rng = np.random.default_rng(29)
    bias = (rng.standard_normal(NH) * 2.0).astype(np.float32)
    C0 = (rng.standard_normal((B, NH, nb, DHV, DHQK)) * 0.2).astype(np.float32)
    n0 = (rng.standard_normal((B, NH)) * 0.5).astype(np.float32)
    m0 = rng.standard_normal((B, NH)).astype(np.float32)
    gd = {"h": Guarded((B, NH, S, DHV), td), "C": Guarded((B, NH, nb, DHV, DHQK), torch.float32),
          "n": Guarded((B, NH), torch.float32), "m": Guarded((B, NH), torch.float32)}
    p = mlstm.fwd_params(B, NH, S, DHQK, DHV, 64, nb, td, False)
    args = [dev(inp[x], td) for x in ("q", "k", "v")] + [dev(inp["igate"]), dev(inp["fgate"]), None, dev(bias),
                                                          dev(C0), dev(n0), dev(m0)]
    with mlstm.bounds_checked() as lib:
        ws = torch.empty(mlstm.scalar_normaliser_workspace_size(p), dtype=torch.uint8, device="cuda")
        st = lib.mlstm_fwd_chunkwise_scalar_normaliser(
            ctypes.byref(p), *[None if a is None else a.data_ptr() for a in args], gd["h"].t.data_ptr(),
            gd["C"].t.data_ptr(), gd["n"].t.data_ptr(), gd["m"].t.data_ptr(), ws.data_ptr(),
            ctypes.c_size_t(ws.numel()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, mlstm.status_string(st)
        st = mlstm.fwd_status(p, ws)
        rec = mlstm.bounds_record(p, ws)
    assert st == 0 and rec == (0, 0, 0), (mlstm.status_string(st), rec)
    assert_guards_intact(gd, "checked scalar normaliser")
    hr, Cr, nr, mr = oracle.sequential_scalar_normaliser(inp["q"], inp["k"], inp["v"], inp["igate"], inp["fgate"],
                                                         bias, None, C0, n0, m0, num_blocks=nb)
    tol = TOL["bf16"]
    errs = {"h": slice_relerr(host(gd["h"].t), hr, 2), "C": slice_relerr(host(gd["C"].t), Cr, 3),
            "n": float(np.max(np.abs(host(gd["n"].t) - nr)) / max(np.max(np.abs(nr)), 1e-30)),
            "m": m_err(host(gd["m"].t), mr)}
    assert all(e <= tol for e in errs.values()), errs


def test_normal_build_reports_no_record():
    """libmlstm.so compiles the checks away; its record call reports nothing."""
    p = mlstm.fwd_params(1, 2, 200, 128, 128, 64, 1, torch.bfloat16, False)
    ws = torch.zeros(mlstm.workspace_size(p), dtype=torch.uint8, device="cuda")
    assert mlstm.lib().mlstm_bounds_checked() == 0
    assert mlstm.bounds_record(p, ws) == (0, 0, 0)


@pytest.mark.parametrize("B,H,T,V", [(2, 3, 200, 128), (1, 2, 130, 64)])
def test_checked_build_gdn2_chunk_finds_no_bad_access(B, H, T, V):
    """The GDN-2 chunk kernels on the tensor cores through the checked build: status OK, an
    empty failure record at bytes 16..39 of the workspace, oracle parity."""
    inp = inputs.gdn2_inputs(B, H, T, 128, V, "bf16", seed=90 + T)
    td = torch.bfloat16
    with mlstm.bounds_checked():
        q, v = dev(inp["q"], td), dev(inp["v"], td)
        ws = torch.zeros(mlstm.gdn2_workspace_size(mlstm.gdn2_params(q, v, "chunk", 64)), dtype=torch.uint8,
                         device="cuda")
        o, S = mlstm.gdn2_fwd(q, dev(inp["k"], td), v, dev(inp["g"]), dev(inp["b"]), dev(inp["w"]), dev(inp["S0"]),
                              mode="chunk", chunk=64, workspace=ws)
        st = mlstm.gdn2_status(q, v, ws)
    rec = ws[16:40].cpu().numpy().view(np.int32)
    assert st == 0 and rec[1] == 0, (mlstm.status_string(st), rec)
    o_ref, S_ref = oracle.gdn2_sequential(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], inp["w"], inp["S0"])
    errs = {"o": slice_relerr(host(o), o_ref, 2), "S": slice_relerr(host(S), S_ref, 2)}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
