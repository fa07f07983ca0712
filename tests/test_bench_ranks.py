"""Host side of the multi-GPU bench path on CPU: two gloo ranks with different step times; the job
time is the slowest rank's and the throughput counts the work of both ranks (weak scaling)."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)

    def reduce_max(x):
        t = torch.tensor([x], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    local_ms = 10.0 + 5.0 * rank          # rank 1 is slower
    ms, value = bench.aggregate_ranks(local_ms, 1e12, world, reduce_max)
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_work(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 10.0 + 5.0 * (world - 1)
    for _, ms, value in res:
        assert ms == slowest
        assert value == pytest.approx(world * 1e12 / (slowest * 1e-3))


def test_single_rank_is_local_time():
    import bench
    ms, value = bench.aggregate_ranks(4.0, 2e12, 1, reduce_max=lambda x: 1e9)
    assert ms == 4.0 and value == pytest.approx(2e12 / 4e-3)


def test_traffic_is_dropped_when_the_kernel_changed(tmp_path, monkeypatch):
    import json
    import bench
    f = tmp_path / "t.json"
    sources = bench.TRAFFIC["append"][1]
    monkeypatch.setitem(bench.TRAFFIC, "append", (str(f), sources))
    f.write_text(json.dumps({"source_sha256_16": bench.source_digest(sources), "bytes_per_launch": 123}))
    assert bench.measured_traffic("append") == 123
    f.write_text(json.dumps({"source_sha256_16": "0" * 16, "bytes_per_launch": 123}))
    assert bench.measured_traffic("append") is None


def test_prepare_bytes_count():
    import bench
    from int8_kv_cache_action_b200.workloads import CONFIGS
    cfg = CONFIGS["C2"]
    # 27680 bf16 rows of K and V (26400 current + 1280 text) x 16 heads x 128: 2 B read + 2 B written each;
    # 15840 history tokens x 16 heads: 2 x 128 codes + 2 scales read, 2 x 128 fp16 + 2 scales written
    want = 27680 * 16 * 128 * 2 * 4 + 15840 * 16 * (2 * 128 + 8 + 4 * 128 + 8)
    assert bench.prepare_bytes(cfg, 15840, 0) == want


def test_reference_arm_line():
    """`bench.py --impl reference` (the timed CPU oracle) prints one JSON line with the measured arm's
    config object, a cpu_baseline describing the sample, and an end-to-end entry with no copies."""
    import json
    import subprocess
    import sys

    import bench
    from int8_kv_cache_action_b200.workloads import CONFIGS
    root = os.path.dirname(os.path.abspath(bench.__file__))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["config"] == bench.step_config(CONFIGS[bench.WORKLOAD], 1)
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True and d["value"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("name", ["C1", "C2", "C4"])
def test_text_row_key_count_matches_the_oracle_mask(name):
    # the bench's algorithmic FLOPs for the text rows count exactly the keys the oracle's rule shows
    import bench
    from int8_kv_cache_action_b200.workloads import CONFIGS
    from oracle import visibility as vis
    cfg = CONFIGS[name]
    frames = sum(p.n_frames for p in cfg.prior)
    lh = (min(frames, cfg.window_frames) if cfg.window_frames else frames) * cfg.tokens_per_frame
    lp = sum(p.head_len for p in cfg.prior)
    m = vis.text_query_mask(lh, lp, cfg.n_query, cfg.tokens_per_frame, cfg.current)
    assert bench.text_key_sum(cfg, lh, lp) == int(m.sum())


def test_dense_attention_launch_count_follows_the_kernel_choice():
    # the bench's launch claim: the production segment runs the pair kernel with a split last wave (two
    # launches: the kernel and the merge of the split units); the 480 x 832 shape runs one block per
    # CTA (one launch); a unit count that is a multiple of the SM count leaves no wave to split
    from bench import dense_attention_launches
    assert dense_attention_launches(26400, 16, 148) == 2       # 1664 pair units, 36 left over
    assert dense_attention_launches(3120, 16, 148) == 1        # pairs take 2 waves against 3 for blocks
    assert dense_attention_launches(148 * 256, 2, 148) == 1    # 148 x 2 units: whole waves only
    assert dense_attention_launches(26400, 16, 132) == 1       # 80 left over of 132: no two shares fit
