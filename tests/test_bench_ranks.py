"""The benchmark's multi-rank host logic on CPU (gloo, world size 2).

Each rank runs an independent problem; the report takes the max of the ranks'
device times and the sum of their work.  No collective touches the data path.
"""
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    r, w, lr = bench.dist_env()
    t = bench.reduce_max(10.0 + 5 * rank, w)
    f = bench.reduce_sum(bench.prefill_flops(1, 32, 1024 * (rank + 1), 128), w)
    q.put((r, w, lr, t, f))
    dist.destroy_process_group()


def test_two_rank_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    want_f = bench.prefill_flops(1, 32, 1024, 128) + bench.prefill_flops(1, 32, 2048, 128)
    for rank, (r, w, lr, t, f) in enumerate(res):
        assert (r, w, lr) == (rank, 2, rank)
        assert t == 15.0
        assert f == want_f


def _failing_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)  # this rank dies before the timing reduction
    try:
        bench.reduce_max(1.0, world)
        q.put("completed")
    except Exception as e:  # noqa: BLE001 - any error is the expected outcome
        q.put(f"error: {type(e).__name__}")


def test_a_dead_rank_ends_the_others_reduction_with_an_error():
    # The survivor's collective fails (peer gone or the short process-group
    # timeout), so the job ends instead of waiting forever.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert procs[1].exitcode == 3
    assert procs[0].exitcode is not None, "surviving rank hung"
    assert q.get(timeout=10).startswith("error")


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.reduce_sum(7.0, 1) == 7.0


def test_work_accounting():
    # 4 * B * Hq * D * L(L+1)/2 at the headline point
    assert bench.prefill_flops(1, 32, 131072, 128) == 4 * 32 * 128 * 131072 * 131073 // 2
    assert bench.decode_bytes(1, 8, 131072, 128) == 2 * 131072 * 8 * 128 * 2
    assert bench.row_flops(32, 128, [0, 9]) == 4 * 32 * 128 * (1 + 10)


def test_reference_arm_line(monkeypatch, capsys):
    # The oracle arm on this machine's cores: one JSON line with the native
    # arm's metric and config, a cpu_baseline describing the run, and an e2e
    # entry with no host-device traffic.  (Run on the tiny workload here, to
    # keep the CPU suite short; the format does not depend on the size.)
    import json
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(bench, "PREFILL_WORKLOAD", "tiny")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                       "--reference-seconds", "8"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.PREFILL_WORKLOAD
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["rows_per_s"] > 0
    assert line["cpu_baseline"]["extrapolated_full_prefill_s"] > 0
    assert line["value"] > 0


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1"]) == 0
    assert capsys.readouterr().out == ""


def test_oracle_rate_extras():
    from zero_shot_rope_bifocal_b200.synth import WORKLOADS
    w = WORKLOADS["qwen3_8b_128k"]
    full = bench.prefill_flops(w.B, w.Hq, w.L, w.D)
    x = bench.oracle_rate_extras(w, full / 1000.0, 2.0, [5, 6, 7, 8])
    assert x["rows_per_s"] == 2.0
    assert abs(x["extrapolated_full_prefill_s"] - 2000.0) < 1e-6


def test_traffic_record_follows_the_kernel_code_not_its_comments(tmp_path, monkeypatch):
    import bench
    src = tmp_path / "k.cu"
    src.write_text("// a comment\n__global__ void k() {}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES", ("k.cu",))
    sha = bench.kernel_sources_sha256()
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", {"bytes": 5.0, "sources_sha256": sha,
                                                  "profile": "p.md"})
    assert bench.measured_traffic() == (5.0, "p.md")
    src.write_text("// another comment\n\n__global__ void k() {}\n")  # comments only
    assert bench.measured_traffic() == (5.0, "p.md")
    src.write_text("// a comment\n__global__ void k() { int x = 1; }\n")  # code changed
    assert bench.measured_traffic()[0] is None

