"""The allocation-free entry point ``attn_run_static`` against the planned path.

``attn_run_static`` is for callers that cannot allocate device memory where they need
attention (an engine that owns all device memory through its own pool, or code running
where allocation is not allowed): it keeps its tables and split-KV scratch in a fixed
array the library reserves per GPU. This file sorts last so a run that stops at the
first failure has already run every other test; it also passes alone in a fresh process.
"""
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import TOL_MAX_ABS, TOL_MEAN_ABS

pytestmark = pytest.mark.gpu


def _batch():
    gen = torch.Generator().manual_seed(3)
    seqs = [W.SeqSpec(20000, 1, W.CAUSAL, []),                 # long enough to be split
            W.SeqSpec(700, 40, W.CAUSAL, []),                  # a causal chunk on a prefix
            W.SeqSpec(300, 1, W.CAUSAL, []),
            W.SeqSpec(2000 + 6, 6, W.TREE, W.random_tree(gen, 6))]
    return W.build_batch("no_alloc", seqs, 32, 8, 128, seed=11, device="cuda")


def _static(b, out):
    return pk.run_static(b.seq_lens, b.query_lens, b.block_table, b.mask_kinds, b.parents_flat,
                         b.q, b.k_cache, b.v_cache, out, num_q_heads=b.num_q_heads,
                         num_kv_heads=b.num_kv_heads, head_dim=b.head_dim,
                         num_pages=b.k_cache.shape[0])


def test_static_entry_point_matches_planned_run_on_two_calls():
    b = _batch()
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_split_units"] > 0          # the split scratch is exercised
    ref = plan.run(b.q, b.k_cache, b.v_cache).clone()
    assert plan.check() == 0
    for _ in range(2):                                   # the array keeps the last call's contents
        out = torch.full_like(b.q, float("nan"))
        _static(b, out)
        torch.cuda.synchronize()
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(d).all()
        assert d.max().item() <= TOL_MAX_ABS and d.mean().item() <= TOL_MEAN_ABS


def test_static_entry_point_rejects_batches_beyond_its_scratch():
    seqs = [W.SeqSpec(1, 1, W.CAUSAL, [])] * 4097       # one more sequence than it holds
    b = W.build_batch("too_many", seqs, 8, 2, 64, seed=1, device="cuda")
    out = torch.empty_like(b.q)
    with pytest.raises(pk.PkvaError) as ei:
        _static(b, out)
    assert ei.value.code == -2 and "static scratch" in str(ei.value)
