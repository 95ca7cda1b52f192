"""The multi-rank host logic of the benchmark, on CPU with the gloo backend and two ranks:
every rank gets its own workload (weak scaling), the step time is the slowest rank's, the
whole-job rate counts every rank's units, and the reference arm runs on rank 0 alone."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    dist = bench.init_dist(world, backend="gloo")
    slowest = bench.max_over_ranks(1.5 * (rank + 1), dist, "cpu")
    work = bench.make_workload("offline_batch", rank, frames=4)
    row = torch.from_numpy(work["enc"]["z"][0, :8].copy())
    rows = [torch.empty_like(row) for _ in range(world)]
    dist.all_gather(rows, row)
    rate = bench.whole_job_rate(work["frames"], world, slowest)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, slowest, [r.tolist() for r in rows], rate))


def test_two_gloo_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, rows, rate in results:
        assert slowest == 3.0                      # the max over ranks, on every rank
        assert rows[0] != rows[1]                  # each rank drew its own workload
        assert rate == pytest.approx(4 * 2 / 3.0e-3)
    assert results[0][2] == results[1][2]          # both ranks saw the same gathered rows


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_roofline_work_per_frame():
    """The roofline's algorithmic work per frame, at every n_q: scores of n_q codebooks of
    2048 x 256 plus the 512 -> 256 projection; n_q int16 codes in and 512 fp32 out for decode."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.enc_flop() == 8 * 2 * 2048 * 256 + 2 * 256 * 512 == 8_650_752
    assert bench.dec_bytes() == 2_064
    for n_q in range(1, 9):
        assert bench.enc_flop(n_q) - bench.enc_flop(n_q - 1) == 2 * 2048 * 256
        assert bench.dec_bytes(n_q) == 2 * n_q + 2048


def test_bench_options():
    """--n-q and --variant reach the encode calls; out-of-range values are refused."""
    run = lambda *a: subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *a],  # noqa: E731
                                    capture_output=True, text=True, timeout=120)
    out = run("--help")
    assert out.returncode == 0 and "--n-q" in out.stdout and "--variant" in out.stdout
    assert run("--n-q", "9").returncode != 0
    assert run("--variant", "2").returncode != 0


def test_world_size_must_match_gpus():
    """--gpus N is never a silent single replica: under torchrun the world must have N ranks;
    without torchrun and N > 1 the script starts the N ranks itself (on 127.0.0.1)."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.check_world(1, {}) == "run"
    assert bench.check_world(8, {}) == "launch"
    assert bench.check_world(4, {"WORLD_SIZE": "4"}) == "run"
    with pytest.raises(SystemExit):
        bench.check_world(8, {"WORLD_SIZE": "1"})
    with pytest.raises(SystemExit):
        bench.check_world(0, {})
    cmd = bench.torchrun_command(["--gpus", "4", "--steps", "3"], 4, 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"] and cmd[-5].endswith("bench.py")
    # a mismatched world exits non-zero before any work
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4",
                        "--impl", "reference", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE=2" in r.stderr


def test_two_part_workload_is_built_from_both_configs():
    """The default step pairs the 1M-frame bf16 encode with the 1M-frame decode-heavy codes,
    each on its own seeded model (shrunk here)."""
    sys.path.insert(0, ROOT)
    import bench
    w = bench.make_workload("encode_decode_1m", 0, frames=16)
    assert w["enc"]["dtype"] == "bf16" and w["enc"]["z"].shape == (16, 512)
    assert w["dec"]["codes"].shape == (16, 8) and not w["decode_own_codes"]
    assert not (w["enc"]["model"].C == w["dec"]["model"].C).all()
    off = bench.make_workload("offline_batch", 0, frames=16)
    assert off["dec"] is None and off["decode_own_codes"]
    assert bench.make_workload("decode_heavy", 0, frames=16)["enc"] is None
