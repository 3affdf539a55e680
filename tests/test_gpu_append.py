"""GPU parity of the fused paged-KV append (attn_run_append): one launch writes the new
tokens' K/V into their cache slots and computes the attention.

Checked on every case:
  * the cache afterwards, bit for bit: the new tokens' slots hold k_new / v_new and every
    other slot is untouched (byte, index work: exact);
  * the output against the float64 oracle (same tolerance as attn_run);
  * the output against attn_run on the cache that already holds the new tokens.
The new tokens' slots start as NaN (the append must never read them) and so do the unused
slots past each sequence's end (no path may let them reach the result).
"""
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, oracle_rows, tc_verify_seqs, tc_verify_wide_seqs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.view(torch.int16)


def run_append_case(b, token_picker=None, seq_ids=None, expect_identical=False):
    tp, ts = W.tail_slots(b)
    exp_k, exp_v = b.k_cache.clone(), b.v_cache.clone()
    exp_k[tp, :, ts] = float("nan")
    exp_v[tp, :, ts] = float("nan")
    k_new, v_new = W.new_token_kv(b)
    pg, sl = W.new_token_slots(b)
    kc, vc = exp_k.clone(), exp_v.clone()
    kc[pg, :, sl] = float("nan")
    vc[pg, :, sl] = float("nan")

    plan = pk.plan_for_batch(b)
    out = plan.run_append(b.q, k_new, v_new, kc, vc)
    assert plan.check() == 0
    assert torch.equal(bits(kc), bits(exp_k)), "k_cache after append"
    assert torch.equal(bits(vc), bits(exp_v)), "v_cache after append"

    rows, exp = oracle_rows(b, seq_ids=seq_ids, token_picker=token_picker)
    assert_close(out[rows], exp, f"{b.name}: append output vs oracle")
    ref = plan.run(b.q, exp_k, exp_v)
    assert plan.check() == 0
    assert_close(ref[rows], exp, f"{b.name}: attn_run (NaN past the end) vs oracle")
    if expect_identical:
        assert torch.equal(bits(out), bits(ref)), "append and attn_run differ on a decode-only batch"
    plan.close()
    return out


@pytest.mark.parametrize("seed, d, max_q", [(11, 64, 9), (12, 128, 40), (13, 128, 6)])
def test_append_small_decode_verify(seed, d, max_q):
    b = W.random_small(seed, num_seqs=6, Hq=16, Hkv=4, d=d, max_ctx=300, max_q=max_q, tree_frac=0.4,
                       device=DEV, bt_extra=2)
    run_append_case(b, expect_identical=True)


@pytest.mark.parametrize("d", [128, 64])
def test_append_prefill_chunks(d):
    """Chunks on the tensor-core prefill path: prefix 0, page- and tile-aligned prefixes,
    ragged ones, a chunk that is not a multiple of the tile, mixed with decode rows."""
    seqs = [W.SeqSpec(300, 300, W.CAUSAL, []),          # no prefix
            W.SeqSpec(128 + 200, 200, W.CAUSAL, []),    # prefix one KV tile
            W.SeqSpec(16 + 64, 64, W.CAUSAL, []),       # prefix one page
            W.SeqSpec(133 + 517, 517, W.CAUSAL, []),    # ragged prefix, three tasks
            W.SeqSpec(7 + 100, 100, W.CAUSAL, []),      # prefix inside the first page
            W.SeqSpec(900, 1, W.CAUSAL, []),
            W.SeqSpec(45, 4, W.TREE, [-1, 0, 0, 2])]
    b = W.build_batch("append_prefill", seqs, 16, 2, d, seed=21, device=DEV, bt_extra=1)
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_prefill_items"] > 0
    plan.close()
    run_append_case(b)


def test_append_mqa_and_mha():
    for Hq, Hkv in ((8, 1), (4, 4)):
        seqs = [W.SeqSpec(77 + 130, 130, W.CAUSAL, []), W.SeqSpec(50, 3, W.CAUSAL, [])]
        b = W.build_batch(f"append_H{Hq}x{Hkv}", seqs, Hq, Hkv, 128, seed=22, device=DEV)
        run_append_case(b)


def _sample(sp):
    T = sp.query_len
    return sorted({0, T // 3, T // 2, T - 1})


def test_append_unified_config_full_size():
    """The mixed prefill / decode / verify batch at its full size, in the benchmark's launch
    configuration: whole cache compared bit for bit, sampled rows against the oracle."""
    b = W.make_config("qwen2_7b_unified", device=DEV)
    seq_ids = list(range(0, len(b.seqs), 7))
    run_append_case(b, token_picker=_sample, seq_ids=seq_ids)


def test_append_prefill_config_two_sequences():
    b = W.make_config("llama33_70b_prefill", device=DEV, max_seqs=2)
    run_append_case(b, token_picker=lambda sp: [0, 127, 128, 1000, sp.query_len - 1], seq_ids=[0, 1])


def test_append_bad_page_is_flagged_not_written():
    seqs = [W.SeqSpec(40, 3, W.CAUSAL, []), W.SeqSpec(20, 20, W.CAUSAL, [])]
    b = W.build_batch("append_bad", seqs, 8, 2, 64, seed=23, device=DEV)
    k_new, v_new = W.new_token_kv(b)
    bt = b.block_table.clone()
    bt[0, 2] = b.k_cache.shape[0] + 5          # the page of positions 32..47: out of range
    plan = pk.Plan(b.seq_lens, b.query_lens, bt, b.mask_kinds, b.parents_flat or None,
                   num_q_heads=8, num_kv_heads=2, head_dim=64, num_pages=b.k_cache.shape[0])
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    plan.run_append(b.q, k_new, v_new, kc, vc)
    assert plan.check() & pk.DEVERR_BAD_PAGE
    # sequence 1 wrote its rows; nothing else changed
    assert torch.equal(bits(kc), bits(b.k_cache)) and torch.equal(bits(vc), bits(b.v_cache))
    plan.close()


def test_append_argument_checks():
    seqs = [W.SeqSpec(40, 3, W.CAUSAL, [])]
    b = W.build_batch("append_args", seqs, 8, 2, 64, seed=24, device=DEV)
    k_new, v_new = W.new_token_kv(b)
    plan = pk.plan_for_batch(b)
    with pytest.raises(ValueError):
        plan.run_append(b.q, k_new[:-1], v_new, b.k_cache, b.v_cache)
    L = pk.lib()
    rc = L.attn_run_append(plan._handle, b.q.data_ptr(), None, v_new.data_ptr(), b.k_cache.data_ptr(),
                           b.v_cache.data_ptr(), b.q.data_ptr(), None)
    assert rc == -1 and b"k_new" in L.attn_last_error()
    plan.close()


def test_append_with_row_split_verify_tasks():
    """A mixed batch whose verify trees (5 tokens x 7 heads = 35 packed rows per KV head) run
    as row-split tasks, one of them split over its long context: the append patches the new
    rows into the pages every consumer warp reads, and one task per (sequence, KV head) writes
    the cache. (head_dim 64: at 128 these trees run as tensor-core tasks, tested below.)"""
    gen = torch.Generator().manual_seed(8)
    seqs = [W.SeqSpec(2500, 1, W.CAUSAL, []) for _ in range(6)] + \
        [W.SeqSpec(9000 + 5, 5, W.TREE, W.random_tree(gen, 5)), W.SeqSpec(300 + 5, 5, W.TREE, W.random_tree(gen, 5))]
    b = W.build_batch("append_row_split", seqs, 28, 4, 64, seed=81, device=DEV)
    items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=28, num_kv_heads=4,
                       head_dim=64, num_pages=b.k_cache.shape[0], bt_stride=b.block_table.shape[1],
                       num_sms=torch.cuda.get_device_properties(0).multi_processor_count, ctas_per_sm=3)
    wide = [it for it in items if it["row_count"] > 16]
    assert wide and any(it["num_splits"] > 1 for it in wide)
    run_append_case(b, expect_identical=True)


def test_append_with_tensor_core_verify_tasks():
    """Verify trees and short causal chunks of 20 to 120 packed rows per KV head run as
    tensor-core tasks over their own keys: under fused append the producers patch the new
    tokens' K / V rows (NaN in the cache beforehand) from the dense input into the tiles, the
    task with the last KV tiles writes them into the cache, and the output is bitwise that of
    attn_run over the appended cache."""
    b = W.build_batch("append_tc_verify", tc_verify_seqs(), 16, 4, 128, seed=83, device=DEV)
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_cascade_items"] > 0
    plan.close()
    run_append_case(b, expect_identical=True)


def test_append_with_tensor_core_verify_tasks_at_the_row_limit():
    """As above with 128-row tensor-core verify tiles (64-node trees under a group of 2), new
    keys across a KV-tile boundary and a causal chunk split into two KV chunks: the patched
    rows span two tiles and the task that writes the cache is the unit's last."""
    b = W.build_batch("append_tc_verify_wide", tc_verify_wide_seqs(), 8, 4, 128, seed=84, device=DEV)
    run_append_case(b, expect_identical=True)
