"""Benchmark: mixed-batch paged attention on B200 through the library's C ABI.

One step = one ``attn_run`` over the unified prefill / decode / verify batch shaped like
Qwen2-7B (28 query / 4 KV heads, head_dim 128, page 16): 4 prefill chunks of 512 tokens,
192 decode sequences (context U[256, 4096]) and 32 verify sequences with a random 5-node
draft tree. Inputs are seeded synthetic bf16 N(0,1) values resident in HBM; the KV cache
(about 1 GB) is larger than L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0). ``--impl reference`` times the float64 CPU oracle on the
host cores on the same workload instead (the reference arm of this benchmark).
Under torchrun each rank runs an independent replica on its own GPU (no data exchange);
timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mixed-batch paged attention: tokens/s; KV GB/s vs HBM peak; prefill TFLOP/s"
DEFAULT_CONFIG = "qwen2_7b_unified"
WORKLOADS = {
    "tiny_decode": "4 decode seqs, ctx {17,64,100,255}, 8q/2kv heads, d64, page 16",
    "llama3_8b_decode": "128 decode seqs, ctx U[512,8192], 32q/8kv heads, d128, page 16",
    "llama33_70b_prefill": "8 x 2048-token causal chunks on ctx U[0,16384], 64q/8kv, d128, page 16",
    "qwen2_7b_unified": "4 x 512 prefill + 192 decode (ctx U[256,4096]) + 32 verify (5-node tree), "
                        "28q/4kv heads, d128, page 16",
    "long_ctx_split": "16 decode seqs, ctx U[32768,131072], 128q/8kv, d128, page 16, 1% outlier keys x8",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.0005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self.period = period_s

    def _run(self):
        nv = self._nv
        stop = self._stop
        while not stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        """Start sampling (again): samples of every entered region accumulate."""
        if self._ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job rate: the units every rank processed, over the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


class OracleRunner:
    """The float64 oracle, as it stands, run over whole sequences of a batch in a cycle.

    Host float64 copies are made up front (not timed); ``run(seconds)`` processes
    sequences in order, wrapping around, until ``seconds`` have elapsed (at least one)."""

    def __init__(self, batch):
        import oracle
        self._oracle = oracle
        self.batch = batch
        self.data = []
        for i, sp in enumerate(batch.seqs):
            k, v = batch.seq_kv(i)
            self.data.append((batch.seq_q(i).double().cpu().numpy(), k.double().cpu().numpy(),
                              v.double().cpu().numpy(), sp))
        self.pos = 0
        self.passes = 0.0
        try:
            import threadpoolctl
            self.threads = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()
                               if i.get("user_api") == "blas")
        except Exception:
            self.threads = len(os.sched_getaffinity(0))

    def run(self, seconds: float):
        tokens, t0 = 0, time.perf_counter()
        while True:
            q, k, v, sp = self.data[self.pos]
            self._oracle.attention([q], [k], [v], [sp.query_len], [sp.mask_kind], [sp.parents])
            tokens += sp.query_len
            self.pos = (self.pos + 1) % len(self.data)
            self.passes += 1.0 / len(self.data)
            el = time.perf_counter() - t0
            if el >= seconds:
                return tokens, el

    def sample_text(self):
        return (f"whole sequences of the same batch taken in order, {self.passes:.2f} passes over "
                f"all {len(self.data)} sequences")


def workload_name(args):
    """The workload as both arms name it (the GPU arm's batch options included)."""
    return f"{args.config}" + (f" (first {args.seqs} sequences)" if args.seqs else "") + \
        (f" ({args.only_class} sequences alone)" if args.only_class else "") + \
        (f" (seed {args.seed})" if args.seed is not None else "") + \
        (" over FP8 E4M3 caches" if args.kv_fp8 else "")


def make_batch(W, args, device):
    """The named configuration's batch with the options both arms apply (first N sequences,
    seed, one class of a mixed batch alone over the same caches)."""
    batch = W.make_config(args.config, device=device, max_seqs=args.seqs, seed=args.seed)
    if args.only_class:
        parts = W.class_batches(batch)
        if args.only_class not in parts:
            raise SystemExit(f"--only-class {args.only_class}: {args.config} has no such sequences")
        batch = parts[args.only_class]
    return batch


def parallelism_text(args, ws, num_kv_heads):
    if ws <= 1:
        return "single GPU"
    if args.shard == "heads":
        from paged_kv_attention_verify_b200 import shard as S
        return "kv-head/sequence shards tp%d x sp%d" % S.shard_layout(ws, num_kv_heads)
    return f"replicas x{ws}"


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import workloads as W
    batch = make_batch(W, args, "cpu")
    runner = OracleRunner(batch)
    step_s = args.ref_seconds / (args.warmup + args.steps)
    for _ in range(args.warmup):
        runner.run(step_s)
    tok, sec = 0, 0.0
    for _ in range(args.steps):
        t, e = runner.run(step_s)
        tok += t
        sec += e
    value = tok / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(args.config, batch, workload_name(args),
                                      parallelism_text(args, ws, batch.num_kv_heads)),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": runner.threads, "kind": "oracle",
                             "sample": "each step: " + runner.sample_text()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "source": source_identity()}
    print(json.dumps(line))
    return 0


def time_steps(plan, batch, out, steps, warmup, stream, ws=1, clk=None, run=None):
    """Device time of `steps` consecutive attn_run calls (one kernel launch each; `run`
    replaces the call), bracketed by a barrier and a synchronize on both sides. Returns
    (per-step ms list, total ms)."""
    import torch
    import torch.distributed as dist
    if run is None:
        def run():
            plan.run(batch.q, batch.k_cache, batch.v_cache, out, stream)
    for _ in range(warmup):
        run()
    if plan.check(stream) != 0:
        raise RuntimeError("device error during warm-up")
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    if clk is not None:
        clk.__enter__()
    try:
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(steps):
            run()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
    finally:
        if clk is not None:
            clk.__exit__()
    if plan.check(stream) != 0:
        raise RuntimeError("device error during the timed region")
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return per, ev[0].elapsed_time(ev[-1])


def time_fn(fn, steps, warmup, stream):
    """Per-step device times (ms) of `steps` calls of fn on `stream` (CUDA events)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]


def _median(xs):
    """Median of per-launch times (ms)."""
    ys = sorted(xs)
    n = len(ys)
    return ys[n // 2] if n % 2 else 0.5 * (ys[n // 2 - 1] + ys[n // 2])


def time_flushed(fn, steps, warmup, stream, flush):
    """Per-step device times (ms) of `steps` calls of fn, each bracketed by its own pair of
    events, with `flush` (a write larger than L2) run before each bracket: for inputs that
    would otherwise stay in L2 from one step to the next."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        flush()
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def roofline(info, seconds, peaks, sustained=False):
    """The binding resource of one launch and how close the launch comes to it.

    HBM: algorithmic K+V bytes (each element once) per launch / launch time.
    Tensor: algorithmic attention flops (4 * D * Hq per allowed query-key pair) / time.
    The bound is whichever takes longer at its measured peak."""
    tf_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_hbm = info["kv_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = info["attn_flops"] / (tf_peak * 1e12)
    if t_hbm >= t_tc:
        ach = info["kv_bytes"] / seconds / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "frac_of_spec_8000": ach / 8000.0}
    ach = info["attn_flops"] / seconds / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": tf_peak, "unit": "TFLOP/s",
            "frac": ach / tf_peak, "frac_of_spec_2250": ach / 2250.0}


def source_identity():
    """The git commit of the checkout (None where the tree carries no .git, as on a copied
    tree) and a SHA-256 over the library's kernel and planner sources."""
    import glob
    import hashlib
    import subprocess
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "paged_kv_attention_verify_b200", "csrc", "*"))):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            h.update(open(f, "rb").read())
    try:
        sha = subprocess.run(["git", "-C", ROOT, "rev-parse", "HEAD"], capture_output=True, text=True,
                             timeout=10).stdout.strip() or None
    except Exception:
        sha = None
    return {"git_sha": sha, "source_sha256": h.hexdigest()}


def workload_config(name, batch, workload_text, parallelism):
    """The ``config`` object of a bench line; both arms print the same one."""
    return {"workload": f"{workload_text}: {WORKLOADS[name]}",
            "query_tokens_per_step": batch.total_q,
            "kv_bytes_per_step": batch_kv_bytes(batch),
            "attn_flops_per_step": batch_attn_flops(batch),
            "l2": "inputs larger than L2 (KV cache read each step exceeds 126 MB)",
            "parallelism": parallelism}


def batch_kv_bytes(batch):
    """Algorithmic K+V bytes of one pass: every cached element of every sequence once."""
    return sum(sp.seq_len for sp in batch.seqs) * batch.num_kv_heads * batch.head_dim * 2 * 2


def batch_attn_flops(batch):
    """Algorithmic attention flops: 4 * D * Hq per allowed (query, key) pair."""
    pairs = 0
    for sp in batch.seqs:
        T, L = sp.query_len, sp.seq_len
        pairs += T * (L - T)
        if sp.mask_kind == 0:
            pairs += T * (T + 1) // 2
        else:
            for i in range(T):                      # a node sees itself and its ancestors
                a, n = i, 0
                while a >= 0:
                    n += 1
                    a = sp.parents[a]
                pairs += n
    return pairs * batch.num_q_heads * 4 * batch.head_dim


def kernel_traffic(workload):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it
    was taken on this workload and on the current kernel sources (else None)."""
    import glob
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")))
    except Exception:
        return None
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "paged_kv_attention_verify_b200", "csrc", "*"))):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            h.update(open(f, "rb").read())
    for e in rec.get("captures", []):
        if e.get("workload") == workload and e.get("source_sha256") == h.hexdigest():
            return e.get("dram_bytes_per_launch")
    return None


def run_ours(args):
    import torch
    import torch.distributed as dist

    import paged_kv_attention_verify_b200 as pk
    import workloads as W

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    batch = make_batch(W, args, dev)
    job_tokens = None
    parallelism = parallelism_text(args, ws, batch.num_kv_heads)
    config = workload_config(args.config, batch, workload_name(args), parallelism)
    if args.shard == "heads" and ws > 1:
        # strong scaling: the one batch split over the ranks (KV-head groups x sequence
        # subsets, no exchange inside attention); every rank builds it from the same seed
        job_tokens = batch.total_q
        batch = W.shard_batch(batch, rank, ws)
        torch.cuda.empty_cache()
    out = torch.empty_like(batch.q)
    run = None
    if args.kv_fp8:
        # the same batch over FP8 (E4M3) caches: attn_plan_kv + attn_run_fp8
        f8 = W.fp8_kv(batch)
        plan = pk.plan_for_batch(batch, kv_fp8=True)

        def run():
            plan.run_fp8(batch.q, f8.k_cache, f8.v_cache_t, f8.k_scale, f8.v_scale, out, stream)
        args.no_e2e = args.no_append = True
    else:
        plan = pk.plan_for_batch(batch)
    info = plan.info()

    clk = ClockSampler(dev.index)
    per, elapsed_ms = time_steps(plan, batch, out, args.steps, args.warmup, stream, ws, clk, run)
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    # end to end through the C ABI with host buffers (pinned), copies inside the region
    e2e_ms = None
    if not args.no_e2e:
        q_host = batch.q.cpu().pin_memory()
        o_host = torch.empty(q_host.shape, dtype=torch.bfloat16).pin_memory()
        # attn_run_host_async: the copy in of step i+1, the attention and the copy out of
        # step i overlap; host_wait orders the closing event after every copy out
        for _ in range(args.warmup):
            plan.run_host_async(q_host, batch.k_cache, batch.v_cache, o_host, stream)
        plan.host_wait(stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        # (no clock sampling here: NVML queries contend with the host-side copies and launches
        # this region times, and cost it a third of its throughput)
        e0.record(stream)
        for _ in range(args.steps):
            plan.run_host_async(q_host, batch.k_cache, batch.v_cache, o_host, stream)
        plan.host_wait(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)

    tokens = batch.total_q
    if job_tokens is not None:       # the ranks share one batch: its tokens over the slowest rank's time
        value = job_tokens * args.steps / (elapsed_ms * 1e-3)
        e2e_value = job_tokens * args.steps / (e2e_ms * 1e-3) if e2e_ms else None
    else:
        value = job_throughput(tokens, args.steps, elapsed_ms, ws)
        e2e_value = job_throughput(tokens, args.steps, e2e_ms, ws) if e2e_ms else None
    avg_launch_s = (sum(per) / len(per)) * 1e-3
    kv_gbs = info["kv_bytes"] / avg_launch_s / 1e9
    tflops = info["attn_flops"] / avg_launch_s / 1e12
    io_bytes = tokens * batch.num_q_heads * batch.head_dim * 2
    workload = workload_name(args)
    rl = roofline(info, avg_launch_s, peaks)
    rl.update({"traffic": kernel_traffic(workload), "kernel": "attn_kernel",
               "peak_source": peaks["source"],
               "per_launch": "algorithmic work of one attn_run (one kernel launch) / its mean CUDA-event time"})
    # fused KV append on the same batch: attn_run_append (one launch that also writes the
    # new tokens' K/V into the cache) against attn_run alone and against a separate scatter
    # (torch index_put) followed by attn_run
    append = None
    if ws == 1 and not args.no_append:
        k_new, v_new = W.new_token_kv(batch)
        pg, sl = W.new_token_slots(batch)
        kc, vc = batch.k_cache, batch.v_cache

        def fused():
            plan.run_append(batch.q, k_new, v_new, kc, vc, out, stream)

        def unfused():
            kc[pg, :, sl] = k_new
            vc[pg, :, sl] = v_new
            plan.run(batch.q, kc, vc, out, stream)

        n = 4 * args.other_steps
        pf = time_fn(fused, n, args.warmup, stream)
        pu = time_fn(unfused, n, args.warmup, stream)
        if plan.check(stream) != 0:
            raise RuntimeError("device error in the append measurement")
        new_bytes = 2 * k_new.numel() * 2                      # K and V of the new tokens
        sf, su = sum(pf) / len(pf) * 1e-3, sum(pu) / len(pu) * 1e-3
        append = {"ms_per_launch": sf * 1e3, "tokens_per_s": tokens / sf,
                  "attn_run_ms": avg_launch_s * 1e3, "scatter_then_attn_run_ms": su * 1e3,
                  "new_kv_bytes": new_bytes,
                  "gbs": (info["kv_bytes"] + 2 * new_bytes) / sf / 1e9,
                  "what": "algorithmic bytes: cache K/V read once + new K/V read and written"}
        del k_new, v_new, pg, sl
    # the batch's classes (prefill chunks, decode steps, verify trees) each timed alone over
    # the same caches, L2 flushed before every launch: where the unified launch's time goes
    # and what running the classes in one launch saves against three launches
    per_class = None
    if ws == 1 and not args.kv_fp8 and not args.no_other_configs:
        parts = W.class_batches(batch)
        if len(parts) > 1:
            per_class = {}
            # the flush writes 512 MB, then reads another 512 MB so that the written lines
            # leave L2 before the timed launch (dirty lines would be written back during it)
            flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
            sweep_buf = torch.zeros(128 << 20, dtype=torch.float32, device=dev)

            def flush():
                flush_buf.fill_(1)
                sweep_buf.sum()
            for cls, b in parts.items():
                pl = pk.plan_for_batch(b)
                inf = pl.info()
                o = torch.empty_like(b.q)

                def step(pl=pl, b=b, o=o):
                    pl.run(b.q, b.k_cache, b.v_cache, o, stream)
                ps = time_flushed(step, args.other_steps, args.warmup, stream, flush)
                if pl.check(stream) != 0:
                    raise RuntimeError("device error in the per-class measurement")
                sec = sum(ps) / len(ps) * 1e-3
                per_class[cls] = {"sequences": len(b.seqs), "query_tokens": b.total_q,
                                  "ms_per_launch": sec * 1e3, "ms_median": _median(ps), "kv_gbs": inf["kv_bytes"] / sec / 1e9,
                                  "attn_tflops": inf["attn_flops"] / sec / 1e12,
                                  "roofline": roofline(inf, sec, peaks)}
                pl.close()
                del b, o
            per_class["sum_of_class_launches_ms"] = sum(v["ms_per_launch"] for v in per_class.values())
            per_class["unified_launch_ms"] = avg_launch_s * 1e3
            del flush_buf, sweep_buf, parts
            torch.cuda.empty_cache()
    plan.close()
    del batch, out

    # the other benchmark batches, same measurement (one launch per step)
    per_config = {}
    if ws == 1 and not args.seqs and not args.only_class and not args.no_other_configs:
        for name in ("llama3_8b_decode", "llama33_70b_prefill", "long_ctx_split"):
            if name == args.config:
                continue
            b = W.make_config(name, device=dev, keep_contiguous=False)
            pl = pk.plan_for_batch(b)
            inf = pl.info()
            o = torch.empty_like(b.q)
            ps, _ = time_steps(pl, b, o, args.other_steps, args.warmup, stream)
            sec = sum(ps) / len(ps) * 1e-3
            per_config[name] = {"ms_per_launch": sec * 1e3, "ms_median": _median(ps), "tokens_per_s": b.total_q / sec,
                                "kv_gbs": inf["kv_bytes"] / sec / 1e9,
                                "attn_tflops": inf["attn_flops"] / sec / 1e12,
                                "roofline": roofline(inf, sec, peaks)}
            pl.close()
            del b, o
            torch.cuda.empty_cache()
        # FP8 (E4M3) caches: the same batches through attn_plan_kv / attn_run_fp8 (decode and
        # verify tasks on the codes, tensor-core tasks on bf16 staging copies made in the same
        # step; algorithmic bytes are the FP8 bytes)
        fp8 = {}
        for name in ("llama3_8b_decode", "long_ctx_split", "qwen2_7b_unified", "llama33_70b_prefill"):
            b = W.make_config(name, device=dev)
            f = W.fp8_kv(b)
            b.k = b.v = None
            torch.cuda.empty_cache()
            pl = pk.plan_for_batch(b, kv_fp8=True)
            inf = pl.info()
            o = torch.empty_like(b.q)

            def step(pl=pl, b=b, f=f, o=o):
                pl.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale, o, stream)

            ps = time_fn(step, args.other_steps, args.warmup, stream)
            if pl.check(stream) != 0:
                raise RuntimeError("device error in the FP8 measurement")
            sec = sum(ps) / len(ps) * 1e-3
            fp8[name] = {"ms_per_launch": sec * 1e3, "ms_median": _median(ps), "tokens_per_s": b.total_q / sec,
                         "kv_bytes_fp8": inf["kv_bytes"], "roofline": roofline(inf, sec, peaks)}
            if name in per_config:
                fp8[name]["speedup_vs_bf16"] = per_config[name]["ms_per_launch"] / (sec * 1e3)
            pl.close()
            del b, f, o
            torch.cuda.empty_cache()
        per_config["fp8_kv"] = fp8
        # shared-prefix batch: cascade plan (attn_plan_shared) against the same batch planned
        # without groups; algorithmic bytes count the shared keys once in both
        for name in W.SHARED_CONFIG_NAMES:
            b = W.make_shared_config(name, device=dev)
            o = torch.empty_like(b.q)
            res = {}
            for tag, shared in (("cascade", True), ("no_cascade", False)):
                pl = pk.plan_for_batch(b, shared=shared)
                inf = pl.info()
                ps, _ = time_steps(pl, b, o, args.other_steps, args.warmup, stream)
                sec = sum(ps) / len(ps) * 1e-3
                res[tag] = {"ms_per_launch": sec * 1e3, "ms_median": _median(ps), "tokens_per_s": b.total_q / sec,
                            "kv_bytes_read_by_plan": inf["kv_bytes"],
                            "cascade_tasks": inf["num_cascade_items"]}
                if shared:
                    kv_unique = inf["kv_bytes"]
                    res[tag]["roofline"] = roofline(inf, sec, peaks)
                pl.close()
            res["kv_bytes_unique"] = kv_unique
            res["speedup"] = res["no_cascade"]["ms_per_launch"] / res["cascade"]["ms_per_launch"]
            # the same groups over FP8 caches (attn_plan_shared_kv + attn_run_fp8: the cascade
            # tasks read bf16 copies of the shared pages staged in the same step)
            f = W.fp8_kv(b)
            pl = pk.plan_for_batch(b, kv_fp8=True)
            inf = pl.info()

            def step8(pl=pl, b=b, f=f, o=o):
                pl.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale, o, stream)

            ps = time_fn(step8, args.other_steps, args.warmup, stream)
            if pl.check(stream) != 0:
                raise RuntimeError("device error in the FP8 shared-prefix measurement")
            sec = sum(ps) / len(ps) * 1e-3
            res["cascade_fp8"] = {"ms_per_launch": sec * 1e3, "ms_median": _median(ps),
                                  "tokens_per_s": b.total_q / sec, "kv_bytes_fp8": inf["kv_bytes"],
                                  "roofline": roofline(inf, sec, peaks),
                                  "speedup_vs_bf16_cascade": res["cascade"]["ms_per_launch"] / (sec * 1e3)}
            pl.close()
            per_config[name] = res
            del b, o, f
            torch.cuda.empty_cache()

    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            b = make_batch(W, args, dev)
            runner = OracleRunner(b)
            tk, sec = runner.run(args.cpu_seconds)
            cpu = {"value": tk / sec, "unit": "tokens/s", "cores": runner.threads, "kind": "oracle",
                   "sample": runner.sample_text()}
            del b
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "ms_median_launch": _median(per), "higher_is_better": True,
            "scaling": "strong" if job_tokens is not None else "weak", "vs_baseline": None,
            "dtype": "bf16 q/out, fp8-e4m3 KV" if args.kv_fp8 else "bf16",
            "data": "synthetic",
            "config": config,
            "kv_gbs": kv_gbs, "kv_frac_of_hbm": kv_gbs / peaks["hbm_gbs"], "prefill_tflops": tflops,
            "roofline": rl,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                    "d2h_bytes_per_step": io_bytes},
            # FP8 plans with tensor-core tasks stage their pages in a launch of its own
            "gpu_launches": args.steps * (2 if args.kv_fp8 and info["num_prefill_items"] > 0 else 1),
            "clocks": clk.summary(),
            "plan": {k: info[k] for k in ("num_decode_items", "num_prefill_items", "num_split_units",
                                          "decode_rows", "kv_bytes", "attn_flops")},
            "source": source_identity(),
            "per_config": per_config,
            "append": append, "per_class": per_class,
        }
        print(json.dumps(result))
    if ws > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--no-append", action="store_true", help="skip the fused KV-append measurement")
    ap.add_argument("--shard", choices=["replica", "heads"], default="replica",
                    help="with N > 1: every rank runs the whole batch (replica, weak scaling) or the batch "
                         "is split over the ranks by KV heads and sequences (heads, strong scaling)")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="time the workload over FP8 E4M3 caches (attn_run_fp8; no e2e or append pass)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the per-config table of the other benchmark batches")
    ap.add_argument("--other-steps", type=int, default=50)
    ap.add_argument("--seqs", type=int, default=None,
                    help="keep only the first N sequences of the batch (smaller profiler captures)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="host time for the oracle baseline line of our arm")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="total host time the reference arm spreads over warm-up + steps")
    ap.add_argument("--only-class", choices=["prefill", "decode", "verify"], default=None,
                    help="time one class of a mixed batch alone over the same caches (profiler captures)")
    ap.add_argument("--seed", type=int, default=None,
                    help="seed of the workload draw (default: the config's index, as the tests use)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
