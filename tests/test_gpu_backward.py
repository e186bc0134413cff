"""GPU parity of the backward (mlstm_bwd, through the C ABI) against the fp64 oracle
(``oracle.sequential_backward``), element by element on the same seeded inputs.

Bounds as for the forward: per (batch, head[, block]) slice, max|x - ref| / max|ref| <= 1e-4
for fp32 inputs and <= 2e-2 for bf16 inputs (gradients are fp32; the oracle sees the same
bf16-rounded values)."""
import math

import numpy as np
import pytest
import torch

import oracle
from linear_recurrent_token_b200 import inputs, mlstm
from tests.helpers import TOL, TORCH_DTYPE, dev, host, slice_relerr

pytestmark = pytest.mark.gpu


def make_case(seed, B, NH, S, DHQK, DHV, nb, dtype, retention, with_state, with_o, with_dstate):
    rng = np.random.default_rng(seed)
    td = TORCH_DTYPE[dtype]

    def rounded(x):  # the values the GPU sees
        return torch.from_numpy(x.astype(np.float32)).to(td).float().numpy().astype(np.float64)

    q = rounded(rng.standard_normal((B, NH, S, DHQK)))
    k = rounded(rng.standard_normal((B, NH, S, DHQK)) / math.sqrt(DHQK / nb))
    v = rounded(rng.standard_normal((B, NH, S, DHV)))
    dh = rounded(rng.standard_normal((B, NH, S, DHV)))
    kw = {}
    if not retention:
        kw["igate"] = rng.standard_normal((B, NH, S)).astype(np.float32).astype(np.float64)
        kw["fgate"] = (rng.standard_normal((B, NH, S)) + 3.0).astype(np.float32).astype(np.float64)
        if with_o:
            kw["ogate"] = rounded(1.0 / (1.0 + np.exp(-rng.standard_normal((B, NH, S, DHV)))))
    dk, dv = DHQK // nb, DHV // nb
    if with_state:
        kw["C0"] = (rng.standard_normal((B, NH, nb, dv, dk)) * 0.3).astype(np.float32).astype(np.float64)
        if not retention:
            kw["n0"] = (rng.standard_normal((B, NH, nb, dk)) * 0.3).astype(np.float32).astype(np.float64)
            kw["m0"] = rng.standard_normal((B, NH)).astype(np.float32).astype(np.float64)
    d = {}
    if with_dstate:
        d["dC"] = rng.standard_normal((B, NH, nb, dv, dk)).astype(np.float32).astype(np.float64)
        if not retention:
            d["dn"] = rng.standard_normal((B, NH, nb, dk)).astype(np.float32).astype(np.float64)
    return q, k, v, dh, kw, d


def run_case(seed, B, NH, S, DHQK, DHV, nb, dtype, retention=False, with_state=False, with_o=False,
             with_dstate=False):
    q, k, v, dh, kw, d = make_case(seed, B, NH, S, DHQK, DHV, nb, dtype, retention, with_state, with_o, with_dstate)
    ref = oracle.sequential_backward(q, k, v, dh, num_blocks=nb, retention=retention, **kw, **d)
    td = TORCH_DTYPE[dtype]
    g = mlstm.bwd(dev(q, td), dev(k, td), dev(v, td), dev(dh, td),
                  dev(kw.get("igate")), dev(kw.get("fgate")),
                  dev(kw.get("ogate"), td) if "ogate" in kw else None,
                  dev(kw.get("C0")), dev(kw.get("n0")), dev(kw.get("m0")), dev(d.get("dC")), dev(d.get("dn")),
                  num_blocks=nb, retention=retention)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    errs = {}
    for key, lead in (("dq", 2), ("dk", 2), ("dv", 2), ("di", 2), ("df", 2), ("do", 2), ("dC0", 3), ("dn0", 3)):
        if ref[key] is None:
            assert g[key] is None, key
            continue
        errs[key] = slice_relerr(host(g[key]), ref[key], lead)
    if ref["dm0"] is not None and with_state:
        dm = host(g["dm0"])
        errs["dm0"] = float(np.max(np.abs(dm - ref["dm0"])) / max(np.max(np.abs(ref["dm0"])), 1e-30))
    bad = {key: e for key, e in errs.items() if not e <= tol}
    assert not bad, f"errors above {tol}: {errs}"
    return errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,NH,S,DHQK,DHV,nb", [
    (1, 2, 40, 16, 16, 1), (2, 2, 33, 32, 64, 2), (1, 3, 70, 64, 32, 1),
])
def test_backward_parity(dtype, B, NH, S, DHQK, DHV, nb):
    run_case(1, B, NH, S, DHQK, DHV, nb, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_parity_with_state_ogate_and_final_state_gradient(dtype):
    run_case(2, 2, 2, 45, 32, 48, 1, dtype, with_state=True, with_o=True, with_dstate=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_parity_retention(dtype):
    run_case(3, 2, 3, 50, 32, 32, 1, dtype, retention=True, with_state=True, with_dstate=True)


def test_backward_parity_block_diagonal_with_state():
    run_case(4, 1, 2, 37, 64, 64, 4, "f32", with_state=True, with_dstate=True)


def test_backward_largest_supported_state():
    # dk = 256, dv = 128: 128 x 257 fp32 of state in shared memory
    run_case(5, 1, 1, 24, 256, 128, 1, "bf16", with_state=True)


def test_backward_empty_sequence_gives_final_state_gradients():
    run_case(6, 2, 2, 0, 16, 16, 1, "f32", with_state=True, with_dstate=True)


def test_backward_workload_sizes_small_blockdiag():
    # the small block-diagonal workload's shapes (B4 NH4 S512 64/64, 2 blocks), bf16
    w = inputs.WORKLOADS[1]
    run_case(7, w.B, w.NH, w.S, w.DHQK, w.DHV, w.num_blocks, w.dtype, with_state=False)


def test_backward_retention_workload_sampled_heads():
    # the retention workload's shapes (64 x 64 per head), a few heads of the batch
    w = inputs.WORKLOADS[2]
    run_case(8, 1, 2, w.S // 4, w.DHQK, w.DHV, 1, w.dtype, retention=True)


# ---------------------------------------------------------------- the cluster kernel
# bf16 blocks of key width 64/128/256 and value width a multiple of 64 up to 512, and narrower
# blocks zero-padded to 64: a thread-block cluster per head, 64 value rows per CTA.
@pytest.mark.parametrize("case", [
    # seed, B, NH, S, DHQK, DHV, nb, retention, with_state, with_o, with_dstate
    (11, 1, 2, 200, 256, 512, 1, False, True, True, True),     # the large-head shape, ragged last chunk
    (12, 1, 1, 96, 256, 512, 1, True, True, False, True),      # retention
    (13, 2, 1, 70, 128, 384, 1, False, False, False, False),   # six CTAs per cluster, no state
    (14, 1, 1, 64, 512, 1024, 2, False, True, True, True),     # two blocks of 256 x 512
    # blocks narrower than 64 keys or values: zero-padded tiles, every global access masked
    (16, 2, 2, 300, 64, 64, 2, False, True, True, True),       # 32 x 32 (the small block-diagonal shape)
    (17, 1, 2, 130, 64, 64, 4, False, True, False, True),      # 16 x 16
    (18, 1, 1, 200, 64, 256, 2, True, True, False, False),     # 32 x 128, retention
    (19, 2, 1, 100, 128, 64, 2, False, True, True, True),      # 64 x 32
    (20, 1, 2, 0, 64, 128, 2, False, True, False, True),       # empty sequence: initial-state gradients
])
def test_backward_cluster_kernel_parity(case):
    seed, B, NH, S, DHQK, DHV, nb, retention, with_state, with_o, with_dstate = case
    run_case(seed, B, NH, S, DHQK, DHV, nb, "bf16", retention=retention, with_state=with_state, with_o=with_o,
             with_dstate=with_dstate)


def test_backward_large_head_workload_sampled_heads():
    """The large-head workload's shapes (256 x 512 per head, bf16), two heads over 1024 tokens
    (the fp64 oracle over the full 8192 x 8 heads would take minutes)."""
    w = inputs.WORKLOADS[3]
    errs = run_case(15, 1, 2, 1024, w.DHQK, w.DHV, 1, w.dtype, with_state=True, with_dstate=True)
    print("large head backward", errs)
