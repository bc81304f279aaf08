"""CPU tests of bench.py's host logic: multi-rank aggregation over gloo
(world size 2) and the reference arm's JSON line."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r pretends to have run 1000 tokens in (1 + r) seconds
        slowest = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        value, t = bench.aggregate_throughput(1000, 1.0 + rank, world, device="cpu")
        q.put((rank, slowest, value, t))
    finally:
        dist.destroy_process_group()


def test_aggregation_over_two_gloo_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value, t in res:
        assert slowest == 2.0 and t == 2.0          # the job's time is the slowest rank's
        assert value == pytest.approx(2 * 1000 / 2.0)  # all ranks' units / that time


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_json_line():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["warmup"] >= 3 and d["steps"] == 1
    assert d["value"] > 0 and d["unit"] == "tokens/s/layer" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_other_ranks_do_no_work():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "1"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_work_accounting_matches_the_hand_counts():
    """The flop and byte counts behind every roofline figure, against counts
    made by hand from the layer shapes: 7B-shaped prefill 828.9 GFLOP of
    GEMMs + 34.4 GFLOP of causal attention per layer; weights per layer
    634.4 MB (13B shape), 1711.3 MB (70B shape), and 7247.8 MB for the 32
    Phi-3-shaped layers."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    W = synth.WORKLOADS
    w7 = W["llama7b_prefill"]
    assert bench.gemm_flops_per_token(w7) * 2048 == pytest.approx(828.9e9, rel=1e-4)
    assert bench.attn_prefill_flops(w7, 1, 2048) == pytest.approx(34.37e9, rel=1e-3)
    # causal pairs: with p0 = 0 the count is L(L+1)/2 per head
    assert bench.attn_prefill_flops(w7, 1, 4) == 4 * 128 * 32 * 10
    assert bench.layer_weight_bytes(W["llama13b_decode"]) == pytest.approx(634.4e6, rel=1e-4)
    assert bench.layer_weight_bytes(W["gqa70b"]) == pytest.approx(1711.3e6, rel=1e-4)
    assert 32 * bench.layer_weight_bytes(W["phi3mini_model"]) == pytest.approx(7247.8e6, rel=1e-4)


def test_gpus_n_starts_n_ranks_itself():
    """``bench.py --gpus 2`` run as a plain command (no torchrun environment)
    starts two ranks itself; with the host-logic fake workload (gloo, no GPU)
    rank r spends (1 + r) ms per step, and the line aggregates both ranks'
    units over the slowest rank's time."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "20",
                        "--warmup", "3", "--fake-workload"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["steps"] == 20
    # both ranks' units over the slowest rank's time: rank 1 sleeps 2 ms per step
    assert d["value"] == pytest.approx(2 * 1000 * 20 / d["slowest_rank_s"])
    assert d["slowest_rank_s"] >= 20 * 0.002
