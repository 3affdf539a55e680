"""Failure detection on the GPU, without faulting it.

* A block-table entry out of range is reported through attn_check (PKVA_EDEVICE with the
  bad-page bit) and its page reads as zeros; the run completes and the other sequences are
  untouched.
* The bounded wait every kernel uses gives up on a barrier nothing completes and reports
  the time-out bit, instead of hanging.
"""
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 300])            # a decode sequence, a prefill chunk
def test_bad_block_table_entry_is_reported_not_faulted(T):
    seqs = [W.SeqSpec(600, T, W.CAUSAL, []), W.SeqSpec(400, 1, W.CAUSAL, [])]
    b = W.build_batch("bad", seqs, 8, 2, 128, seed=4, device="cuda")
    bt = b.block_table.clone()
    bt[0, 3] = b.k_cache.shape[0] + 1000            # out of range (the sequence has 38 pages)
    plan = pk.Plan(b.seq_lens, b.query_lens, bt, b.mask_kinds, None, num_q_heads=8, num_kv_heads=2,
                   head_dim=128, num_pages=b.k_cache.shape[0])
    out = plan.run(b.q, b.k_cache, b.v_cache)
    bits = plan.check()
    assert bits & pk.DEVERR_BAD_PAGE
    assert torch.isfinite(out.float()).all()
    # sequence 1 does not use the bad entry: still exact
    rows, exp = oracle_rows(b, [1])
    assert_close(out[rows], exp, "untouched sequence")
    assert plan.check() == 0                         # attn_check cleared the word


@pytest.mark.parametrize("T", [1, 300])            # FP8: a decode task, or the bf16 staging pass
def test_bad_block_table_entry_fp8_and_cascade(T):
    """The same report on the FP8 path and on a shared-prefix (cascade) plan."""
    seqs = [W.SeqSpec(600, T, W.CAUSAL, []), W.SeqSpec(400, 1, W.CAUSAL, [])]
    b = W.build_batch("bad8", seqs, 8, 2, 128, seed=5, device="cuda")
    f = W.fp8_kv(b)
    bt = b.block_table.clone()
    bt[0, 3] = -7                                   # negative: out of range too
    plan = pk.Plan(b.seq_lens, b.query_lens, bt, b.mask_kinds, None, num_q_heads=8, num_kv_heads=2,
                   head_dim=128, num_pages=b.k_cache.shape[0], kv_fp8=True)
    out = plan.run_fp8(b.q, f.k_cache, f.v_cache_t, f.k_scale, f.v_scale)
    assert plan.check() & pk.DEVERR_BAD_PAGE
    assert torch.isfinite(out.float()).all()
    plan.close()
    sb = W.random_shared_small(6, 16, 4, device="cuda")
    bt = sb.block_table.clone()
    bt[0, 1] = sb.k_cache.shape[0]                  # a shared page of group 0, seen by its cascade tasks
    plan = pk.Plan(sb.seq_lens, sb.query_lens, bt, sb.mask_kinds, sb.parents_flat, num_q_heads=16,
                   num_kv_heads=4, head_dim=128, num_pages=sb.k_cache.shape[0],
                   prefix_group=sb.prefix_group, prefix_len=sb.prefix_len)
    out = plan.run(sb.q, sb.k_cache, sb.v_cache)
    assert plan.check() & pk.DEVERR_BAD_PAGE
    assert torch.isfinite(out.float()).all()
    plan.close()


def test_bounded_wait_gives_up_with_timeout_bit():
    assert pk.selftest_wait_timeout(20_000_000) == pk.DEVERR_TIMEOUT
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
