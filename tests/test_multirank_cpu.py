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


def test_kernel_traffic_record(tmp_path, monkeypatch):
    """bench.py takes a kernel's DRAM traffic per launch from the committed ncu record
    (a JSON file), and only while the record's source hash matches the kernel source."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    committed = json.load(open(bench.TRAFFIC_FILE))
    for key, rec in committed.items():
        kernel, workload = key.split("@")
        assert isinstance(rec["traffic_bytes_per_launch"], int)
        assert len(rec["kernel_source_sha1"]) == 40 and rec["command"]
    sha = bench._source_sha1()
    f = tmp_path / "t.json"
    f.write_text(json.dumps({"prep@w": {"traffic_bytes_per_launch": 123,
                                        "kernel_source_sha1": sha, "command": "x"},
                             "chain@w": {"traffic_bytes_per_launch": 456,
                                         "kernel_source_sha1": "0" * 40, "command": "x"}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.kernel_traffic("prep", "w") == 123
    assert bench.kernel_traffic("chain", "w") is None      # taken on another build
    assert bench.kernel_traffic("fused", "w") is None      # no record


def test_kernel_bytes_and_flops():
    """The algorithmic accounting of the bench line, on the 35B-A3B layer shape: bytes
    of the whole call and of each kernel, and the chunk form's tensor flops."""
    sys.path.insert(0, ROOT)
    import bench
    T, N, H_qk, H_v, d = 4096, 1, 16, 32, 128
    call = bench.prefill_bytes(T, N, H_qk, H_v, d, 2, False)
    assert call == 103_809_024
    assert bench.kernel_bytes("fused_half_rows", T, N, H_qk, H_v, d, 2, False) == call
    assert bench.kernel_bytes("chain", T, N, H_qk, H_v, d, 2, False) == call - 8 * T * H_v
    assert bench.kernel_bytes("prep", T, N, H_qk, H_v, d, 2, False) == \
        4 * T * H_qk * d + 8 * T * H_v
    # H_qk 4 C d + H_v (2 C d + 4 C d + 6 d^2) per token
    assert bench.prefill_flops(T, N, H_qk, H_v, d) == 21_474_836_480
