"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerance (bf16 inputs, fp32 accumulation, bf16 output): max abs <= 2e-2 and mean abs
<= 2e-3 per compared set of rows. Small batches are compared on every row; the
full-size batches on sampled sequences and tokens, in the launch configuration the
benchmark times.
"""
import numpy as np
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, oracle_rows, tc_verify_seqs, tc_verify_wide_seqs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_batch(b, plan=None):
    plan = plan or pk.plan_for_batch(b)
    out = plan.run(b.q, b.k_cache, b.v_cache)
    assert plan.check() == 0
    return out, plan


def test_tiny_decode_config_all_rows():
    b = W.make_config("tiny_decode", device=DEV)
    out, plan = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, "tiny_decode")
    assert plan.info()["num_decode_items"] > 0


SMALL = [
    dict(seed=1, Hq=8, Hkv=2, d=64, max_ctx=80, max_q=40),
    dict(seed=2, Hq=8, Hkv=2, d=128, max_ctx=300, max_q=20),
    dict(seed=3, Hq=28, Hkv=4, d=128, max_ctx=500, max_q=12, tree_frac=0.6),
    dict(seed=4, Hq=16, Hkv=16, d=128, max_ctx=200, max_q=33),
    dict(seed=5, Hq=32, Hkv=2, d=64, max_ctx=700, max_q=5, tree_frac=0.5),
    dict(seed=6, Hq=4, Hkv=1, d=128, max_ctx=40, max_q=64, tree_frac=0.5, max_draft=64),
    dict(seed=7, Hq=64, Hkv=8, d=128, max_ctx=2000, max_q=9, num_seqs=5),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: f"seed{c['seed']}_H{c['Hq']}x{c['Hkv']}_d{c['d']}")
def test_small_mixed_batches_all_rows(cfg):
    cfg = dict(cfg)
    b = W.random_small(cfg.pop("seed"), device=DEV, bt_extra=3, **cfg)
    out, _ = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, "small batch")


@pytest.mark.parametrize("cfg", SMALL[:5], ids=lambda c: f"fma_seed{c['seed']}")
def test_cuda_core_body_small_batches(cfg, monkeypatch):
    """The CUDA-core page body (kept for comparison) against the oracle too."""
    monkeypatch.setenv("PKVA_DECODE_BODY", "fma")
    cfg = dict(cfg)
    b = W.random_small(cfg.pop("seed"), device=DEV, bt_extra=3, **cfg)
    out, _ = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, "small batch, CUDA-core body")


def test_edge_lengths():
    """ctx 1, ctx at a page boundary, page + 1, a query longer than a page, a 64-node tree."""
    seqs = [W.SeqSpec(1, 1, W.CAUSAL, []), W.SeqSpec(16, 1, W.CAUSAL, []),
            W.SeqSpec(17, 1, W.CAUSAL, []), W.SeqSpec(32, 32, W.CAUSAL, []),
            W.SeqSpec(48, 17, W.CAUSAL, []),
            W.SeqSpec(64 + 3, 64, W.TREE, W.random_tree(torch.Generator().manual_seed(5), 64)),
            W.SeqSpec(5, 5, W.TREE, [-1, 0, 0, 1, 3])]
    for d in (64, 128):
        b = W.build_batch("edges", seqs, 8, 2, d, seed=77, device=DEV)
        out, _ = run_batch(b)
        rows, exp = oracle_rows(b)
        assert_close(out[rows], exp, f"edges d{d}")


def test_page_permutation_gives_bitwise_identical_output():
    b1 = W.random_small(21, num_seqs=5, Hq=16, Hkv=4, d=128, max_ctx=900, max_q=10, device=DEV)
    b2 = W.repage(b1, perm_seed=4242)
    assert not torch.equal(b1.block_table, b2.block_table)
    o1, _ = run_batch(b1)
    o2, _ = run_batch(b2)
    assert torch.equal(o1, o2)


def test_repeated_runs_are_identical_and_reset_split_state():
    b = W.build_batch("long", [W.SeqSpec(20000, 1, W.CAUSAL, []), W.SeqSpec(9000, 3, W.TREE, [-1, 0, 0])],
                      32, 2, 128, seed=3, device=DEV)
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_split_units"] > 0
    o1 = plan.run(b.q, b.k_cache, b.v_cache).clone()
    o2 = plan.run(b.q, b.k_cache, b.v_cache)
    assert torch.equal(o1, o2)
    rows, exp = oracle_rows(b)
    assert_close(o2[rows], exp, "split")


def test_decode_steps_match_prefill_rows_on_gpu():
    L, T = 300, 24
    full = W.build_batch("pf", [W.SeqSpec(L, T, W.CAUSAL, [])], 8, 2, 128, seed=9, device=DEV)
    o_full, _ = run_batch(full)
    k, v = full.seq_kv(0)
    for i in (0, 7, 23):
        Li = L - T + i + 1
        step = W.build_batch("st", [W.SeqSpec(Li, 1, W.CAUSAL, [])], 8, 2, 128, seed=9, device=DEV)
        step.q = full.q[i:i + 1].clone()
        # same keys/values, laid out in the step batch's own pool
        step.k_cache.zero_()
        step.v_cache.zero_()
        P = 16
        for pos in range(Li):
            pg = step.block_table[0, pos // P].item()
            step.k_cache[pg, :, pos % P] = k[pos]
            step.v_cache[pg, :, pos % P] = v[pos]
        o_step, _ = run_batch(step)
        d = (o_step[0].float() - o_full[i].float()).abs().max().item()
        assert d <= 2e-2, (i, d)


def test_run_host_matches_run():
    b = W.random_small(31, num_seqs=6, Hq=8, Hkv=2, d=128, max_ctx=400, max_q=8, device=DEV)
    plan = pk.plan_for_batch(b)
    o_dev = plan.run(b.q, b.k_cache, b.v_cache)
    q_host = b.q.cpu().pin_memory()
    o_host = torch.empty(q_host.shape, dtype=torch.bfloat16).pin_memory()
    plan.run_host(q_host, b.k_cache, b.v_cache, o_host)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(o_host, o_dev.cpu())


def test_run_host_back_to_back_calls():
    """Successive host calls alternate staging buffers and overlap the next copy of q with
    the previous attention; each output must still match its own q (prefill tasks included,
    so the q tensor map changes between calls)."""
    seqs = [W.SeqSpec(300, 200, W.CAUSAL, []), W.SeqSpec(90, 1, W.CAUSAL, []), W.SeqSpec(45, 4, W.TREE, [-1, 0, 0, 1])]
    b = W.build_batch("host_calls", seqs, 16, 2, 128, seed=44, device=DEV)
    plan = pk.plan_for_batch(b)
    qs = [(b.q.float() * f).to(torch.bfloat16) for f in (1.0, -0.5, 2.0, 0.25, 1.5)]
    refs = [plan.run(q, b.k_cache, b.v_cache).cpu() for q in qs]
    q_hosts = [q.cpu().pin_memory() for q in qs]
    o_hosts = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for q in qs]
    for qh, oh in zip(q_hosts, o_hosts):
        plan.run_host(qh, b.k_cache, b.v_cache, oh)
    torch.cuda.current_stream().synchronize()
    assert plan.check() == 0
    for i, (oh, ref) in enumerate(zip(o_hosts, refs)):
        assert torch.equal(oh, ref), i


def test_run_host_async_pipelined_calls():
    """attn_run_host_async: copies out on the plan's own stream, two out buffers; after
    host_wait and a synchronize every output matches its own q."""
    seqs = [W.SeqSpec(300, 200, W.CAUSAL, []), W.SeqSpec(90, 1, W.CAUSAL, []), W.SeqSpec(45, 4, W.TREE, [-1, 0, 0, 1])]
    b = W.build_batch("host_async", seqs, 16, 2, 128, seed=45, device=DEV)
    plan = pk.plan_for_batch(b)
    qs = [(b.q.float() * f).to(torch.bfloat16) for f in (1.0, -0.5, 2.0, 0.25, 1.5, -1.0)]
    refs = [plan.run(q, b.k_cache, b.v_cache).cpu() for q in qs]
    q_hosts = [q.cpu().pin_memory() for q in qs]
    o_hosts = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for q in qs]
    stream = torch.cuda.current_stream()
    for qh, oh in zip(q_hosts, o_hosts):
        plan.run_host_async(qh, b.k_cache, b.v_cache, oh, stream)
    plan.host_wait(stream)
    stream.synchronize()
    assert plan.check() == 0
    for i, (oh, ref) in enumerate(zip(o_hosts, refs)):
        assert torch.equal(oh, ref), i


def test_run_rejects_misaligned_pointer():
    b = W.make_config("tiny_decode", device=DEV)
    plan = pk.plan_for_batch(b)
    L = pk.lib()
    rc = L.attn_run(plan._handle, b.q.data_ptr() + 2, b.k_cache.data_ptr(), b.v_cache.data_ptr(),
                    b.q.data_ptr(), None)
    assert rc == -1


FULL = ["llama3_8b_decode", "qwen2_7b_unified", "long_ctx_split", "llama33_70b_prefill"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_config_sampled(name):
    """The full-size batches in the launch configuration the benchmark times, against the
    oracle on: every sequence of the 70B prefill batch at the tile and task boundaries
    (tokens 0, 127 / 128, 255 / 256, 511 / 512 and the last), every sequence of the
    long-context batch, 32 of the Llama-3-8B decode sequences, and on the unified batch every
    prefill chunk at its boundaries, every verify tree and 32 decode sequences."""
    b = W.make_config(name, device=DEV)
    out, plan = run_batch(b)
    n = len(b.seqs)
    picker = None
    if name == "llama33_70b_prefill":
        seq_ids = list(range(n))
        picker = lambda sp: [0, 127, 128, 255, 256, 511, 512, sp.query_len - 1]
    elif name == "qwen2_7b_unified":
        kinds = [W.seq_class(sp) for sp in b.seqs]
        pre = [i for i, k in enumerate(kinds) if k == "prefill"]
        ver = [i for i, k in enumerate(kinds) if k == "verify"]
        dec = [i for i, k in enumerate(kinds) if k == "decode"]
        rows, exp = oracle_rows(b, pre, lambda sp: [0, 127, 128, 255, 256, sp.query_len - 1])
        assert_close(out[rows], exp, f"{name} prefill chunks")
        seq_ids = ver + dec[::len(dec) // 32][:32]
    elif name == "long_ctx_split":
        seq_ids = list(range(n))
    else:
        seq_ids = list(range(0, n, n // 32))[:32]
    rows, exp = oracle_rows(b, seq_ids, picker)
    assert_close(out[rows], exp, name)
    # every output row is finite
    assert torch.isfinite(out.float()).all()


def test_unified_batch_classes_alone():
    """Each class of the unified Qwen2-7B-shaped batch (prefill chunks, decode steps, verify
    trees) planned and run alone over the shared caches, as the benchmark times them."""
    b = W.make_config("qwen2_7b_unified", device=DEV)
    parts = W.class_batches(b)
    assert sorted(parts) == ["decode", "prefill", "verify"]
    for cls, p in parts.items():
        out, plan = run_batch(p)
        info = plan.info()
        if cls == "prefill":
            assert info["num_prefill_items"] > 0 and info["num_decode_items"] == 0
        else:
            assert info["num_prefill_items"] == 0 and info["num_decode_items"] > 0
        n = len(p.seqs)
        seq_ids = sorted({0, n // 2, n - 1})
        picker = (lambda sp: [0, 1, 255, 256, sp.query_len - 1]) if cls == "prefill" else None
        rows, exp = oracle_rows(p, seq_ids, picker)
        assert_close(out[rows], exp, f"qwen2_7b_unified[{cls}]")
        plan.close()


@pytest.mark.parametrize("Hq, Hkv", [(16, 4), (28, 4), (32, 2)])
def test_tensor_core_verify_tasks_all_rows(Hq, Hkv):
    """Rows of 17 to 128 per KV head with at least 512 keys run as tensor-core tasks over their
    own keys (one pass for all rows, the two warpgroups' halves of the KV tiles combined),
    including KV chunks merged as split partials; every row against the oracle, and a second
    run is bitwise the same. With 28 / 4 and 32 / 2 heads some units exceed 128 rows and stay
    on the decode/verify path beside them."""
    b = W.build_batch("tc_verify", tc_verify_seqs(), Hq, Hkv, 128, seed=94, device=DEV)
    items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=Hq,
                       num_kv_heads=Hkv, head_dim=128, num_pages=b.k_cache.shape[0],
                       bt_stride=b.block_table.shape[1],
                       num_sms=torch.cuda.get_device_properties(0).multi_processor_count, ctas_per_sm=3)
    assert any(it["kind"] == 2 for it in items)
    out, plan = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, f"tensor-core verify Hq={Hq} Hkv={Hkv}")
    again = plan.run(b.q, b.k_cache, b.v_cache)
    assert plan.check() == 0
    assert torch.equal(out, again)


def test_tensor_core_verify_tasks_wide_trees_and_chunks():
    """Tensor-core verify tasks at their limits: 64-node trees under a group of 2 (128 packed
    rows, ancestor bits across all four 32-column mask words), one with its new keys across a
    KV-tile boundary, a 63-token causal chunk (126 rows) split into two chunks of KV tiles,
    and a 40-node chain; every row against the oracle."""
    b = W.build_batch("tc_verify_wide", tc_verify_wide_seqs(), 8, 4, 128, seed=95, device=DEV)
    items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=8,
                       num_kv_heads=4, head_dim=128, num_pages=b.k_cache.shape[0],
                       bt_stride=b.block_table.shape[1],
                       num_sms=torch.cuda.get_device_properties(0).multi_processor_count, ctas_per_sm=3)
    assert {it["seq"] for it in items if it["kind"] == 2} == {12, 13, 14, 15}
    assert any(it["kind"] == 2 and it["num_splits"] > 1 for it in items)
    out, plan = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, "tensor-core verify, 128-row tiles")
    plan.close()


@pytest.mark.parametrize("seed", range(200, 216))
def test_random_mixed_batches_with_tensor_core_verify(seed):
    """Random mixed batches at head_dim 128 (4 to 13 sequences, contexts up to 3000 keys,
    trees of up to 32 nodes, causal chunks of up to 40 tokens, six head shapes): where verify
    units qualify and are a minority of the pages they run as tensor-core verify tasks,
    elsewhere on the decode/verify path. Every row against the oracle."""
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv = [(8, 2), (16, 4), (28, 4), (32, 8), (8, 4), (32, 2)][seed % 6]
    ns = int(torch.randint(4, 14, (1,), generator=g))
    b = W.random_small(seed, num_seqs=ns, Hq=Hq, Hkv=Hkv, d=128,
                       max_ctx=int(torch.randint(300, 3000, (1,), generator=g)),
                       max_q=int(torch.randint(2, 40, (1,), generator=g)), tree_frac=0.6,
                       max_draft=int(torch.randint(2, 33, (1,), generator=g)), device=DEV, bt_extra=1)
    out, plan = run_batch(b)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, f"random mixed batch {seed}")


def test_row_split_verify_tasks_all_rows():
    """Verify trees of 35 and 48 packed rows per KV head among decode steps run as row-split
    tasks (one warp streams each page once, three own 16 rows each), split over long contexts
    and not; trees of 80 and 96 rows (group 16) as a 48-row task plus 16-row or 48-row ones.
    Every row against the oracle, and a second run is bitwise the same."""
    gen = torch.Generator().manual_seed(9)
    seqs = [W.SeqSpec(3000 + 7 * i, 1, W.CAUSAL, []) for i in range(8)] + \
        [W.SeqSpec(12000 + 5, 5, W.TREE, W.random_tree(gen, 5)), W.SeqSpec(600 + 5, 5, W.TREE, W.random_tree(gen, 5)),
         W.SeqSpec(37 + 6, 6, W.TREE, W.random_tree(gen, 6))]
    for Hq, Hkv in ((28, 4), (32, 2)):        # 35 / 42 rows; 80 / 96 rows (48-row tasks plus 16-row ones)
        # head_dim 64: at 128 the longer trees run as tensor-core tasks instead
        b = W.build_batch("row_split", seqs, Hq, Hkv, 64, seed=91, device=DEV)
        items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=Hq,
                           num_kv_heads=b.num_kv_heads, head_dim=64, num_pages=b.k_cache.shape[0],
                           bt_stride=b.block_table.shape[1],
                           num_sms=torch.cuda.get_device_properties(0).multi_processor_count, ctas_per_sm=3)
        assert any(it["row_count"] > 16 for it in items)
        out, plan = run_batch(b)
        rows, exp = oracle_rows(b)
        assert_close(out[rows], exp, f"row-split Hq={Hq} Hkv={Hkv}")
        again = plan.run(b.q, b.k_cache, b.v_cache)
        assert plan.check() == 0
        assert torch.equal(out, again)
