"""The N > 1 host logic of bench.py on CPU with two gloo ranks: the
max-over-ranks timing reduction, and the reference arm's rank gating
(rank 0 alone runs and prints; other ranks exit 0 without work)."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.5, 7.25][rank]
        q.put((rank, bench.max_over_ranks(local_ms)))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 7.25, 1: 7.25}


def test_max_over_ranks_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5) == 2.5


def test_reference_arm_runs_on_rank_zero_only():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen(
            [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
             "--workload", "tiny", "--steps", "3", "--warmup", "3", "--ref-budget-s", "2"],
            env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=300) for p in procs]
    assert [p.returncode for p in procs] == [0, 0], [o[1][-2000:] for o in outs]
    line = json.loads(outs[0][0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert outs[1][0].strip() == ""
    # the reference arm reports the same config object as our arm would
    sys.path.insert(0, ROOT)
    import bench
    assert line["config"] == bench.config_of(bench.get_workload("tiny"), 2)


def test_gpus_n_without_torchrun_relaunches_as_n_ranks():
    # started as one plain process, --gpus 2 must run two ranks (torchrun,
    # gloo-free here: the reference arm needs no process group) and print one line
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    p = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
         "--workload", "tiny", "--steps", "3", "--warmup", "3", "--ref-budget-s", "2"],
        env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_must_match_world_size():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, timeout=300)
    assert p.returncode != 0 and "WORLD_SIZE" in p.stderr


def test_bench_work_accounting():
    sys.path.insert(0, ROOT)
    import bench
    import moe_synth
    cfg = moe_synth.get_config("qwen3_decode")
    counts = [4] * 120 + [0] * 8
    w = bench.work_per_step(cfg, counts)
    assert w["active_experts"] == 120
    assert w["weight_bytes"] == 120 * 3 * 2048 * 768 * 2
    assert w["layer_flops"] == 2 * 64 * 8 * 3 * 2048 * 768
    assert bench.launches_per_step(cfg) == 2          # counter reset, the persistent decode kernel
    assert w["fused"]["bytes"] == w["weight_bytes"] + 64 * 2048 * 2 * 2 + 64 * 128 * 4
    assert bench.launches_per_step(moe_synth.get_config("qwen3_decode", T=65)) == 5   # route, permute, 2 GEMMs, finalize
    assert bench.launches_per_step(moe_synth.get_config("qwen3_prefill")) == 7
    q = moe_synth.get_config("w4a16_decode")
    wq = bench.work_per_step(q, [8] * 256)
    assert wq["weight_bytes"] == 256 * (2 * 2048 * (7168 // 2 + 56 * 2) + 7168 * (2048 // 2 + 16 * 2))


def test_bench_rejects_too_few_warmup_steps():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])


def test_stored_traffic_follows_its_kernel_sources(tmp_path, monkeypatch):
    """A profile summary's DRAM figure is reported while the files it names
    hash as stored, and dropped (None) once they do not."""
    sys.path.insert(0, ROOT)
    import bench
    files = ["common.cuh", "launch_util.cuh"]
    h = bench.kernel_source_hash([f"{bench.CSRC_DIR}/{n}" for n in files])
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    body = "dram_bytes_per_launch: 12345\nkernel_sources: {}\nkernel_source_sha256_16: {}\n"
    (tmp_path / "k_w.md").write_text(body.format(" ".join(files), h))
    assert bench.profiled_traffic("k", "w") == 12345.0
    (tmp_path / "k_w.md").write_text(body.format(" ".join(reversed(files)), h))   # other files, other hash
    assert bench.profiled_traffic("k", "w") is None
    (tmp_path / "k_w.md").write_text(body.format("no_such_file.cu", h))
    assert bench.profiled_traffic("k", "w") is None
    assert bench.profiled_traffic("k", "missing") is None
    # the committed summaries of the graded workloads carry a source list
    for name in ("gemm_swiglu_qwen3_prefill", "gemm_swiglu_skewed", "gemm_swiglu_w4a16_decode", "fused_qwen3_decode"):
        text = open(os.path.join(ROOT, "profiles", name + ".md")).read()
        assert "kernel_sources:" in text and "kernel_source_sha256_16:" in text
