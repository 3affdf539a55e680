"""The allocation-free entry point ``attn_run_static`` against the oracle and the planned path.

``attn_run_static`` is for callers that cannot allocate device memory where they need
attention (an engine that owns all device memory through its own pool, or code running
where allocation is not allowed): it keeps its tables and split-KV scratch in a fixed
array the library reserves per GPU. This file sorts last so a run that stops at the
first failure has already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import TOL_MAX_ABS, TOL_MEAN_ABS, assert_close, oracle_rows

pytestmark = pytest.mark.gpu


def _batch(d=128, Hq=32, Hkv=8, seed=11):
    gen = torch.Generator().manual_seed(3)
    seqs = [W.SeqSpec(20000, 1, W.CAUSAL, []),                 # long enough to be split
            W.SeqSpec(700, 40, W.CAUSAL, []),                  # a causal chunk on a prefix
            W.SeqSpec(300, 1, W.CAUSAL, []),
            W.SeqSpec(2000 + 6, 6, W.TREE, W.random_tree(gen, 6))]
    return W.build_batch("no_alloc", seqs, Hq, Hkv, d, seed=seed, device="cuda")


def _static(b, out):
    return pk.run_static(b.seq_lens, b.query_lens, b.block_table, b.mask_kinds, b.parents_flat,
                         b.q, b.k_cache, b.v_cache, out, num_q_heads=b.num_q_heads,
                         num_kv_heads=b.num_kv_heads, head_dim=b.head_dim,
                         num_pages=b.k_cache.shape[0])


def _two_calls_match(b):
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_split_units"] > 0          # the split scratch is exercised
    ref = plan.run(b.q, b.k_cache, b.v_cache).clone()
    assert plan.check() == 0
    rows, exp = oracle_rows(b)
    for _ in range(2):                                   # the array keeps the last call's contents
        out = torch.full_like(b.q, float("nan"))
        _static(b, out)
        torch.cuda.synchronize()
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(d).all()
        assert d.max().item() <= TOL_MAX_ABS and d.mean().item() <= TOL_MEAN_ABS
        assert_close(out[rows], exp, "attn_run_static against the oracle")


def test_static_entry_point_matches_planned_run_and_oracle_on_two_calls():
    _two_calls_match(_batch())


def test_static_entry_point_head_dim_64_split_case():
    _two_calls_match(_batch(d=64, Hq=16, Hkv=4, seed=12))


def test_static_entry_point_rejects_batches_beyond_its_scratch():
    seqs = [W.SeqSpec(1, 1, W.CAUSAL, [])] * 4097       # one more sequence than it holds
    b = W.build_batch("too_many", seqs, 8, 2, 64, seed=1, device="cuda")
    out = torch.empty_like(b.q)
    with pytest.raises(pk.PkvaError) as ei:
        _static(b, out)
    assert ei.value.code == -2 and "static scratch" in str(ei.value)


def test_static_entry_point_rejects_split_partials_beyond_its_scratch():
    # 128 sequences x 8 KV heads of 1025 pages each: the per-task page cap (1024) splits every
    # unit in two, 2048 partial slots against the 1024 the scratch holds at head_dim 128, and
    # coarser plans cannot lower that. The block table aliases a small pool of pages (only
    # planning runs: the call is rejected before any launch).
    B, Hq, Hkv, D, pages = 128, 32, 8, 128, 1025
    pool = 64
    bt = (torch.arange(B * pages, dtype=torch.int32) % pool).reshape(B, pages).cuda()
    kc = torch.zeros(pool, Hkv, 16, D, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(pk.PkvaError) as ei:
        pk.run_static([pages * 16] * B, [1] * B, bt, [W.CAUSAL] * B, None, q, kc, kc, out, num_q_heads=Hq,
                      num_kv_heads=Hkv, head_dim=D, num_pages=pool)
    assert ei.value.code == -2 and "split partials" in str(ei.value)


def test_static_entry_point_rejects_memory_off_the_current_device():
    # through the C ABI directly: an output in page-locked host memory is refused before
    # anything is launched
    b = _batch()
    host_out = torch.empty(b.q.shape, dtype=torch.bfloat16).pin_memory()
    sl, ql, mk, par = pk._host_arrays(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat)
    rc = pk.lib().attn_run_static(len(sl), pk._ptr(sl), pk._ptr(ql), b.block_table.data_ptr(),
                                  b.block_table.shape[1], b.k_cache.shape[0], pk._ptr(mk), pk._ptr(par),
                                  b.num_q_heads, b.num_kv_heads, b.head_dim, 16, ctypes.c_float(0.0),
                                  b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(),
                                  host_out.data_ptr(), None)
    assert rc == -1 and b"out" in pk.lib().attn_last_error()


def test_static_binding_checks_shapes_and_dtypes():
    b = _batch()
    out = torch.empty_like(b.q)
    bad = [dict(q=b.q[:-1]), dict(out=out.float()), dict(k_cache=b.k_cache[:, :4]),
           dict(block_table=b.block_table.long()), dict(out=torch.empty_like(b.q).transpose(0, 1))]
    for over in bad:
        args = dict(q=b.q, out=out, k_cache=b.k_cache, block_table=b.block_table)
        args.update(over)
        with pytest.raises(ValueError):
            pk.run_static(b.seq_lens, b.query_lens, args["block_table"], b.mask_kinds, b.parents_flat,
                          args["q"], args["k_cache"], b.v_cache, args["out"], num_q_heads=b.num_q_heads,
                          num_kv_heads=b.num_kv_heads, head_dim=b.head_dim, num_pages=b.k_cache.shape[0])
