"""Host-side logic of bench.py: work accounting and the multi-rank (replica) timing path.

The multi-rank path is exercised with world_size 2 on the gloo backend on the CPU:
every rank contributes its own time and the slowest one is reported.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import oracle


def test_chunkwise_flop_count_matches_hand_count():
    # large-head workload: (L+1)(dk+dv) + 4 dk dv + 4 dk per token and head
    per_tok = 65 * 768 + 4 * 256 * 512 + 4 * 256
    assert per_tok == 575_232
    assert bench.chunkwise_flops(1, 8, 8192, 256, 512, 64) == 8 * 8192 * per_tok
    # retention drops the normaliser term
    assert bench.chunkwise_flops(1, 1, 1, 64, 64, 64, retention=True) == 65 * 128 + 4 * 64 * 64


def test_decode_bytes_are_dominated_by_the_state_stream():
    b = bench.decode_step_bytes(128, 8, 256, 512, 2)
    state_c = 128 * 8 * 256 * 512 * 4 * 2
    assert state_c == 1_073_741_824
    assert b == 1_079_001_088
    assert state_c / b > 0.99


def test_state_bytes_context_number():
    assert oracle.state_bytes(32, 8, 256, 512, 2) == 67_240_448


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, wsz, local = bench.dist_setup(world)
    assert (r, wsz, local) == (rank, world, rank)
    bench.dist_barrier(wsz)
    slow = bench.dist_max(1.5 + rank, wsz)
    out[rank] = slow
    import torch.distributed as dist
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_report_the_slowest_rank():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_recorded_traffic_is_null_once_sources_change(monkeypatch):
    import bench
    key = ("tc_walk", "large_head")
    rec = dict(bench.RECORDED_TRAFFIC[key])
    monkeypatch.setitem(bench.RECORDED_TRAFFIC, key, dict(rec, sha256="0" * 64))
    assert bench.recorded_traffic(*key) is None
    monkeypatch.setitem(bench.RECORDED_TRAFFIC, key, dict(rec, sha256=bench.sources_sha256(rec["sources"])))
    assert bench.recorded_traffic(*key) == rec["bytes"]
    assert bench.recorded_traffic("tc_walk", "retention") is None


def test_backward_flop_count_and_simt_peak():
    # six dk x dv products / rank-1 updates per token and block, 2 flops per element
    assert bench.backward_flops(1, 1, 1, 64, 32, 1) == 6 * 2 * 64 * 32
    assert bench.backward_flops(4, 4, 512, 32, 32, 2) == 4 * 4 * 512 * 2 * 12 * 32 * 32
    assert abs(bench.fp32_simt_peak_tflops(1965.0) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9


def _fake_gdn2(rank):
    ms_p, ms_c, ms_d = 2.0 + rank, 4.0 + 2 * rank, 0.1 * (1 + rank)
    tokens, flops, nbytes = 1000.0, 9e9, 5e8
    alu = lambda ms: {"bound": "alu", "achieved": flops / (ms * 1e-3) / 1e12, "peak": 1.0, "unit": "TFLOP/s",
                      "frac": 0.0, "traffic": None}
    return {"gdn2_prefill": {"workload": "w", "recurrent": {"value": tokens / (ms_p * 1e-3), "unit": "tokens/s",
                                                            "ms_per_step": ms_p, "roofline": alu(ms_p)},
                             "chunk": {"value": tokens / (ms_c * 1e-3), "unit": "tokens/s", "ms_per_step": ms_c,
                                       "roofline": alu(ms_c)}},
            "gdn2_decode": {"workload": "d", "value": nbytes / (ms_d * 1e-3) / 1e9, "unit": "GB/s",
                            "ms_per_step": ms_d, "tokens_per_s": 256 / (ms_d * 1e-3),
                            "roofline": {"bound": "hbm", "achieved": nbytes / (ms_d * 1e-3) / 1e9, "peak": 6535.4,
                                         "unit": "GB/s", "frac": 0.0, "traffic": None}},
            "steps": 5}


def _gdn2_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    bench.dist_setup(world)
    out[rank] = bench.gdn2_over_ranks(_fake_gdn2(rank), world, 1965.0)
    import torch.distributed as dist
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_gdn2_leg_reports_the_slowest_rank_and_the_job_throughput():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_gdn2_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    rec = res[0]["gdn2_prefill"]["recurrent"]
    assert rec["ms_per_step"] == 3.0 and abs(rec["value"] - 2 * 1000 / 3e-3) < 1e-6 * rec["value"]
    assert abs(rec["roofline"]["peak"] - bench.fp32_simt_peak_tflops(1965.0)) < 1e-9
    assert abs(rec["roofline"]["achieved"] - 9e9 / 3e-3 / 1e12) < 1e-9
    assert res[0]["gdn2_prefill"]["chunk"]["ms_per_step"] == 6.0
    dec = res[0]["gdn2_decode"]
    assert abs(dec["ms_per_step"] - 0.2) < 1e-12 and abs(dec["value"] - 2 * 5e8 / 0.2e-3 / 1e9) < 1e-6
    assert abs(dec["roofline"]["achieved"] - 5e8 / 0.2e-3 / 1e9) < 1e-6 and dec["roofline"]["peak"] == 6535.4
    # one rank: unchanged times and values
    one = bench.gdn2_over_ranks(_fake_gdn2(0), 1, 1965.0)
    assert one["gdn2_prefill"]["recurrent"]["ms_per_step"] == 2.0
    assert abs(one["gdn2_prefill"]["recurrent"]["value"] - 1000 / 2e-3) < 1e-6


def test_gdn2_inputs_follow_their_recipe():
    from linear_recurrent_token_b200 import inputs
    x = inputs.gdn2_inputs(2, 3, 50, 16, 8, "bf16", seed=1)
    import numpy as np
    assert x["q"].shape == (2, 3, 50, 16) and x["v"].shape == (2, 3, 50, 8) and x["S0"].shape == (2, 3, 16, 8)
    np.testing.assert_allclose(np.linalg.norm(x["k"], axis=-1), 1.0, rtol=1e-2)  # unit keys (bf16-rounded)
    assert np.all(x["g"] < 0) and np.all((x["b"] >= 0) & (x["b"] <= 1)) and np.all((x["w"] >= 0) & (x["w"] <= 1))
    # stored values are exact in the storage type
    import torch
    assert np.array_equal(torch.from_numpy(x["q"]).to(torch.bfloat16).float().numpy(), x["q"])
    assert inputs.gdn2_inputs(1, 1, 3, 8, 8, "f32", seed=1, with_state=False)["S0"] is None


def test_gdn2_flop_count():
    # decay K V, read-out 2 K V, erase + write 4 K V, output 2 K V per token and head
    assert bench.gdn2_flops(1, 1, 1, 128, 128) == 9 * 128 * 128
    assert bench.gdn2_flops(8, 16, 2048, 128, 128) == 38_654_705_664


def test_reference_arm_runs_on_rank_zero_only():
    """Under a launcher with several ranks, `bench.py --impl reference` prints its line from rank
    0 alone; any other rank exits 0 without work and prints nothing."""
    import subprocess
    import sys

    from tests.conftest import ROOT
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
