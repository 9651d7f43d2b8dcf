"""Host logic of the multi-GPU bench path, on CPU: world-size-2 gloo ranks.

The data path has no collective (each rank quantizes and multiplies its own
token shard with replicated weights); the only cross-rank steps are the
timing reductions (max over ranks) and rank 0 printing the job's line."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        # each rank measured its own time; the job takes the slowest rank's
        local = [10.0 + 5.0 * rank, 3.0 - rank, 7.5]
        agg = bench.max_over_ranks(local, w, dist, "cpu")
        e2e = bench.max_over_ranks([1.0 + rank], w, dist, "cpu")
        q.put((r, w, lr, agg, e2e))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, w, lr, agg, e2e) in enumerate(out):
        assert (r, w, lr) == (rank, 2, rank)
        assert agg == [15.0, 3.0, 7.5]   # element-wise max over the two ranks
        assert e2e == [2.0]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2.0], 1) == [1.5, 2.0]


def test_job_throughput_is_weak_scaling():
    ops, steps = 2.0 * 8192 * 1152 * 3456, 20
    one = bench.job_throughput(ops, steps, 1, 1.0)
    # same per-rank time on 4 ranks -> 4x the job's throughput
    assert bench.job_throughput(ops, steps, 4, 1.0) == pytest.approx(4 * one)
    # the slowest rank sets the job's time
    assert bench.job_throughput(ops, steps, 4, 2.0) == pytest.approx(2 * one)
    assert one == pytest.approx(ops * steps / 1e-3 / 1e12)


def test_each_rank_gets_its_own_token_shard():
    cfg = synth.CONFIGS[1].with_tokens(64)
    seeds = [bench.shard_seed(cfg, r) for r in range(8)]
    assert len(set(seeds)) == 8
    x0 = synth.make_x(cfg, seed=seeds[0])
    x1 = synth.make_x(cfg, seed=seeds[1])
    assert x0.shape == x1.shape and not np.array_equal(x0, x1)
    w0, _ = synth.make_w(cfg)
    w1, _ = synth.make_w(cfg)
    assert np.array_equal(w0, w1)  # replicated weights


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_roofline_traffic_only_while_kernel_unchanged(tmp_path):
    """bench.py reports an ncu DRAM-traffic figure only while the kernel's
    sources still hash to the value recorded beside it."""
    csrc = tmp_path / "hadamard_rotated_bit_token_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES["gemm"]:
        (csrc / f).write_text(f"// {f}\n")
    (tmp_path / "profiles").mkdir()
    name = bench.PROFILES[("gemm", 2)]
    digest = bench.kernel_source_hash("gemm", str(tmp_path))
    (tmp_path / "profiles" / name).write_text(
        f"summary\n\n    traffic_bytes_per_launch: 12345\n    kernel_source_sha256: {digest}\n")
    assert bench.profiled_traffic("gemm", 2, str(tmp_path)) == 12345
    assert bench.profiled_traffic("gemm", 3, str(tmp_path)) is None      # no summary
    (csrc / "hq_gemm.cu").write_text("// changed\n")
    assert bench.profiled_traffic("gemm", 2, str(tmp_path)) is None      # stale summary
