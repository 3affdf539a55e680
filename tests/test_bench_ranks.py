"""The multi-rank plumbing of bench.py on CPU with gloo (world size 2): the job's time is
the slowest rank's, throughput counts every rank's units, and the reference arm runs on
rank 0 only (the other ranks exit 0 without work or output). Each rank of the GPU
benchmark is an independent replica, so no data crosses ranks."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ws, r, local = bench.dist_env()
    slow = bench.max_over_ranks(10.0 + 5.0 * rank)          # rank 1 is the slow one
    q.put((r, ws, local, slow, bench.job_throughput(100, 4, slow, ws)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, ws, local, slow, thr) in enumerate(res):
        assert (r, ws, local) == (rank, 2, rank)
        assert slow == 15.0                                  # the slowest rank's time
        assert thr == pytest.approx(2 * 100 * 4 / 15e-3)     # all ranks' units / that time


def test_single_process_defaults():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(10, 2, 4.0, 1) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    """Rank 0 (single process): one JSON line with the arm's keys; the oracle on host cores,
    no host-device traffic."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--ref-seconds", "2"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]
    # the same config object the GPU arm prints for this workload
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    b = W.make_config(bench.DEFAULT_CONFIG)
    assert d["config"] == bench.workload_config(bench.DEFAULT_CONFIG, b, bench.DEFAULT_CONFIG, "single GPU")
    assert d["source"]["source_sha256"]


def test_bench_algorithmic_counts_match_the_oracle_masks():
    """The bench's algorithmic flop count (4 * D * Hq per allowed query-key pair) against the
    number of allowed pairs the oracle's masks give, on a batch with causal chunks and trees."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import workloads as W
    b = W.random_small(5, num_seqs=8, Hq=8, Hkv=2, d=64, max_ctx=60, max_q=20, tree_frac=0.5)
    pairs = 0
    for sp in b.seqs:
        m = oracle.allowed_mask(sp.seq_len, sp.query_len, sp.mask_kind, sp.parents or None)
        pairs += int(m.sum())
    assert bench.batch_attn_flops(b) == pairs * b.num_q_heads * 4 * b.head_dim
    assert bench.batch_kv_bytes(b) == sum(sp.seq_len for sp in b.seqs) * b.num_kv_heads * b.head_dim * 4


def test_only_class_keeps_one_class_over_the_same_caches():
    """``--only-class`` times one class of the mixed batch alone: the batch keeps only that
    class's sequences (their query rows and block-table rows) over the same page pool, and
    both arms name the workload with the class."""
    import argparse
    import torch
    import bench
    import workloads as W
    full = W.make_config(bench.DEFAULT_CONFIG)
    for cls in ("prefill", "decode", "verify"):
        args = argparse.Namespace(config=bench.DEFAULT_CONFIG, seqs=None, seed=None, only_class=cls, kv_fp8=False)
        b = bench.make_batch(W, args, "cpu")
        keep = [i for i, sp in enumerate(full.seqs) if W.seq_class(sp) == cls]
        assert keep and [sp.seq_len for sp in b.seqs] == [full.seqs[i].seq_len for i in keep]
        assert b.k_cache.shape == full.k_cache.shape
        assert torch.equal(b.block_table, full.block_table[keep])
        assert b.q.shape[0] == sum(full.seqs[i].query_len for i in keep)
        assert f"({cls} sequences alone)" in bench.workload_name(args)
    args = argparse.Namespace(config="llama3_8b_decode", seqs=None, seed=None, only_class="verify", kv_fp8=False)
    with pytest.raises(SystemExit):
        bench.make_batch(W, args, "cpu")
