"""Host-side logic of the multi-GPU benchmark path, run as 2 gloo ranks on CPU:
independent per-rank seeds, max-over-ranks timing, rank-0-only output."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist = bench.init_dist(world, "gloo")
    r, w, _ = bench.dist_env()
    assert (r, w) == (rank, world)
    m = bench.max_over_ranks(dist, 10.0 + rank)
    bench.barrier(dist)
    out[rank] = (m, bench.rank_seed(3, rank))
    dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0
    assert out[0][1] != out[1][1]


def test_single_process_is_identity():
    assert bench.max_over_ranks(None, 3.5) == 3.5
    bench.barrier(None)


def test_reference_arm_other_ranks_exit(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert capsys.readouterr().out == ""


def test_traffic_record_tracks_kernel_source(tmp_path, monkeypatch):
    f = tmp_path / "t.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", f)
    assert bench.recorded_traffic() is None
    f.write_text(f"kernel_source_sha256_16: {bench.source_digest(bench.BWD_SOURCE)}\n"
                 "dram_bytes_per_full_launch: 12345\n")
    assert bench.recorded_traffic() == 12345
    f.write_text("kernel_source_sha256_16: 0000\ndram_bytes_per_full_launch: 12345\n")
    assert bench.recorded_traffic() is None


@pytest.mark.parametrize("argv", [["--workload", "c2", "--window", "10"], ["--bias-mode", "alibi"],
                                  ["--with-backward"], ["--num-splits", "4"]])
def test_options_outside_their_workload_are_rejected(argv):
    with pytest.raises(SystemExit):
        bench.check_args(bench.parse_args(argv))


def test_options_on_their_workload_are_accepted():
    for argv in (["--window", "1024"], ["--workload", "c4", "--bias-mode", "alibi"],
                 ["--workload", "c5a", "--with-backward"], ["--workload", "kv1", "--num-splits", "8"]):
        bench.check_args(bench.parse_args(argv))


def test_source_digest_ignores_comments_but_not_code(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("int f(int x) { return x + 1; }\n")
    b.write_text("// a note\nint f(int x) {  /* the increment */\n  return x + 1;  // plus one\n}\n")
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench.source_digest(a) == bench.source_digest(b)
    assert bench.source_digest(a) != bench.source_digest(c)
