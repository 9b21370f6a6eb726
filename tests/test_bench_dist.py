"""Host-side logic of the multi-GPU benchmark path, on CPU with gloo and two
ranks: every rank runs its own (b, h) shard (no data-path collective); the job
time is the slowest rank's and the value counts all ranks' work."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t_max = bench.max_over_ranks(times[rank], world)
        value = bench.weak_scaling_value(world, 1.0e12, 10, t_max)
        out[rank] = (t_max, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    times = [120.0, 180.0]            # ms of the timed region per rank
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), times, out), nprocs=world, join=True)
    for rank in range(world):
        t_max, value = out[rank]
        assert t_max == 180.0
        # 2 ranks x 10 steps x 1 TFLOP in 0.18 s
        assert value == pytest.approx(2 * 10 * 1.0 / 0.18)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(1, 2e12, 5, 1000.0) == pytest.approx(10.0)


def test_kernel_table_shares_and_flops():
    w = bench.workload_cfg(bench.parse_args([]))
    t = bench.kernel_table([("fa_fwd_kernel", 1.0), ("fa_bwd_dkdv_kernel", 2.0),
                            ("fa_bwd_dq_kernel", 1.0)], w)
    assert t["fa_bwd_dkdv_kernel"]["share"] == pytest.approx(0.5)
    f1 = 4.0 * 32 * 8192 * 8192 * 128 / 2
    assert t["fa_fwd_kernel"]["algorithmic_tflops"] == pytest.approx(f1 / 1e-3 / 1e12)
    assert t["fa_bwd_dkdv_kernel"]["algorithmic_tflops"] == pytest.approx(2 * f1 / 2e-3 / 1e12)


def test_sweep_overrides_name_and_batch():
    w = bench.workload_cfg(bench.parse_args(["--workload", "sweep", "--seq-len", "2048", "--causal", "0"]))
    assert (w["B"], w["Nq"], w["Nk"], w["causal"]) == (8, 2048, 2048, False)
    assert w["name"] == "sweep-H16-N2048-full"      # stored ncu traffic never matches it
    w = bench.workload_cfg(bench.parse_args(["--workload", "sweep", "--seq-len", "32768"]))
    assert (w["B"], w["Nq"]) == (1, 32768)          # B = max(1, 16384 // N)
    with pytest.raises(SystemExit):
        bench.workload_cfg(bench.parse_args(["--workload", "llama", "--seq-len", "512"]))


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # bench reports ncu DRAM bytes only while the kernel's own source file and
    # the shared device headers hash to the revision the capture was taken from
    csrc = tmp_path / "exact_attention_112_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "fa_bwd.cu").write_text("// backward v1\n")
    (csrc / "fa_fwd.cu").write_text("// forward v1\n")
    (csrc / "fa_ptx.cuh").write_text("// primitives v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rev = bench.kernel_rev("fa_bwd_dkdv_kernel")
    import json
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"fa_bwd_dkdv_kernel:llama": {"kernel_rev": rev, "bytes_per_launch": 123}}))
    w = {"name": "llama"}
    assert bench.load_traffic("fa_bwd_dkdv_kernel", w) == 123
    assert bench.load_traffic("fa_fwd_kernel", w) is None
    assert bench.load_traffic("fa_bwd_dkdv_kernel", {"name": "bwd"}) is None
    (csrc / "fa_fwd.cu").write_text("// forward v2\n")        # another kernel's file
    (csrc / "fa_new.cu").write_text("// a new file\n")
    assert bench.load_traffic("fa_bwd_dkdv_kernel", w) == 123
    (csrc / "fa_ptx.cuh").write_text("// primitives v2\n")    # a shared header
    assert bench.kernel_rev("fa_bwd_dkdv_kernel") != rev
    assert bench.load_traffic("fa_bwd_dkdv_kernel", w) is None
    (csrc / "fa_ptx.cuh").write_text("// primitives v1\n")
    (csrc / "fa_bwd.cu").write_text("// backward v2\n")       # the kernel's own file
    assert bench.load_traffic("fa_bwd_dkdv_kernel", w) is None
