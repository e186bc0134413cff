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
