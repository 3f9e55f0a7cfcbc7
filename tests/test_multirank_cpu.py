"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each), as torchrun
launches them. Every (sequence, V head) unit is independent, so ranks run replicas with
no data-path collective; the only collectives are the barrier and the max over ranks of
the timings, checked here."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    from linear_attention_sequence_delta_b200.inputs import make_prefill_inputs

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench._dist()
        bench._barrier(w)
        # each rank times its own replica; the job's time is the slowest rank's
        mx = bench._max_over_ranks(1.0 + 2.0 * r, w, "cpu")
        # replicas draw different inputs (seed = rank)
        P = make_prefill_inputs([8], H_qk=1, H_v=2, d_k=64, d_v=64, seed=r)
        gathered = [torch.zeros_like(P.q) for _ in range(w)]
        dist.all_gather(gathered, P.q)
        out[r] = (w, r, local, mx, not torch.equal(gathered[0], gathered[1]))
        bench._barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ws = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(ws, _free_port(), out), nprocs=ws, join=True,
                       start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(ws):
        w, rank, local, mx, differ = out[r]
        assert (w, rank, local) == (ws, r, r)
        assert mx == 3.0          # max over ranks of 1 + 2 r
        assert differ             # each replica has its own inputs


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(2.5, 1, "cpu") == 2.5
    bench._barrier(1)


def test_kernel_profile_lines_parse():
    """bench.py reads the dominant kernel's DRAM traffic and the source hash it was taken on
    from the committed ncu summary (list-marked lines)."""
    sys.path.insert(0, ROOT)
    import bench
    traffic, sha = bench._kernel_traffic()
    assert isinstance(traffic, int) and 10**7 < traffic < 10**9
    assert isinstance(sha, str) and len(sha) == 40 and all(c in "0123456789abcdef" for c in sha)
    assert len(bench._kernel_source_sha1()) == 40
