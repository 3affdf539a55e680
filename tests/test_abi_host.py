"""Host-side checks of the C ABI (no GPU): the library loads, exports every entry point
the header declares, validates its inputs, and the planner's tile tasks cover the batch
exactly once."""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_attention_verify_b200 as pk
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "pkva.h")).read()
    return sorted(set(re.findall(r"PKVA_API\s+[\w\s\*]*?\b((?:attn|pkva)_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = pk.lib()
    syms = header_symbols()
    assert len(syms) >= 8
    assert set(syms) == set(pk.EXPORTED)
    for s in syms:
        assert hasattr(L, s), s


def _plan_args(**over):
    a = dict(seq_lens=[40, 17], query_lens=[8, 1], mask_kind=[W.CAUSAL, W.CAUSAL], parents=None,
             num_q_heads=8, num_kv_heads=2, head_dim=64, num_pages=8, bt_stride=4)
    a.update(over)
    return a


def _inspect(**over):
    a = _plan_args(**over)
    return pk.inspect(a.pop("seq_lens"), a.pop("query_lens"), a.pop("mask_kind"), a.pop("parents"), **a)


@pytest.mark.parametrize("over, code", [
    (dict(query_lens=[0, 1]), -1),                          # query_len = 0
    (dict(query_lens=[41, 1]), -1),                         # query_len > seq_len
    (dict(seq_lens=[0, 17], query_lens=[0, 1]), -1),        # empty sequence
    (dict(num_q_heads=6, num_kv_heads=4), -1),              # Hq not a multiple of Hkv
    (dict(head_dim=96), -2),                                # unsupported head_dim
    (dict(bt_stride=2), -1),                                # block table too narrow
    (dict(mask_kind=[2, 0]), -1),                           # unknown mask kind
    (dict(mask_kind=[W.TREE, 0], parents=None), -1),        # tree without parents
    (dict(mask_kind=[W.TREE, 0], parents=[-1, 0, 1, 3, 0, 0, 0, 0]), -1),  # parent not earlier
    (dict(mask_kind=[W.TREE, 0], parents=[-1, 0, -2, 0, 0, 0, 0, 0]), -1), # parent < -1
    (dict(seq_lens=[100, 17], query_lens=[65, 1], mask_kind=[W.TREE, 0],
          parents=[-1] * 65, bt_stride=8), -1),             # tree too large
])
def test_planner_rejects_bad_batches(over, code):
    with pytest.raises(pk.PkvaError) as ei:
        _inspect(**over)
    assert ei.value.code == code
    assert pk.lib().attn_last_error().decode()


def test_attn_plan_validates_before_touching_the_device():
    # a non-NULL block-table pointer that is never dereferenced: validation fails first
    L = pk.lib()
    h = ctypes.c_void_p()
    sl = (ctypes.c_int32 * 1)(5)
    ql = (ctypes.c_int32 * 1)(6)
    mk = (ctypes.c_int32 * 1)(0)
    rc = L.attn_plan(ctypes.byref(h), 1, sl, ql, ctypes.c_void_p(0x1000), 1, 1, mk, None, 8, 2, 64, 16, 0.0)
    assert rc == -1 and not h.value
    assert b"query_lens" in L.attn_last_error()
    rc = L.attn_plan(ctypes.byref(h), 1, sl, sl, None, 1, 1, mk, None, 8, 2, 64, 16, 0.0)
    assert rc == -1 and b"block_table" in L.attn_last_error()
    assert L.attn_run(None, None, None, None, None, None) == -1
    assert L.attn_check(None, None, None) == -1
    L.attn_plan_destroy(None)


def _tc_verify_set(batch, head_dim=128, prefix_group=None, prefix_len=None):
    """Sequences whose rows run as tensor-core verify tasks over all of their keys: outside any
    caller group, 17 to 128 packed rows per KV head, at least 512 keys, and together at most
    half of the decode/verify pages of the batch (otherwise none)."""
    G = batch.num_q_heads // batch.num_kv_heads
    cand, own_pages, all_pages = set(), 0, 0
    for s, sp in enumerate(batch.seqs):
        if sp.mask_kind == W.CAUSAL and sp.query_len >= 64:       # a prefill chunk
            continue
        grouped = prefix_group is not None and prefix_group[s] >= 0
        pages = (sp.seq_len + 15) // 16 - (prefix_len[prefix_group[s]] // 16 if grouped else 0)
        all_pages += pages
        if head_dim == 128 and not grouped and 16 < sp.query_len * G and sp.query_len <= 128 // G and \
                sp.seq_len >= 512:
            cand.add(s)
            own_pages += pages
    return cand if 2 * own_pages <= all_pages else set()


def _shared_keys(batch, s, prefix_group, prefix_len, head_dim=128):
    """Keys of sequence s that cascade-kind tasks cover: its group's shared prefix, or all keys
    of a tensor-core verify sequence (no decode/verify task)."""
    if prefix_group is not None and prefix_group[s] >= 0:
        return prefix_len[prefix_group[s]]
    return batch.seqs[s].seq_len if s in _tc_verify_set(batch, head_dim, prefix_group, prefix_len) else 0


def _coverage(batch, items, prefix_group=None, prefix_len=None, head_dim=128):
    """Every (seq, kv head, packed row) must see exactly the keys it needs, once."""
    G = batch.num_q_heads // batch.num_kv_heads
    q_start = np.cumsum([0] + [sp.query_len for sp in batch.seqs])
    shared = [_shared_keys(batch, s, prefix_group, prefix_len, head_dim) for s in range(len(batch.seqs))]
    seen = {}
    for it in items:
        assert it["key_begin"] % 16 == 0 and it["key_end"] > it["key_begin"]
        if it["kind"] == 1:            # prefill: tokens [row_begin, +row_count) of one query head
            assert 1 <= it["row_count"] <= 256 and it["q_head"] // G == it["kv_head"]
            rows = [(it["seq"], t * G + it["q_head"] % G)
                    for t in range(it["row_begin"], it["row_begin"] + it["row_count"])]
        elif it["kind"] == 2:          # cascade: all heads of q rows [row_begin, +row_count)
            assert it["q_head"] == -1 and 1 <= it["row_count"] <= 2 * (128 // G)
            rows = []
            for tok in range(it["row_begin"], it["row_begin"] + it["row_count"]):
                s = int(np.searchsorted(q_start, tok, side="right") - 1)
                if prefix_group is not None and prefix_group[s] >= 0:
                    assert prefix_group[s] == prefix_group[it["seq"]]
                else:                  # a single-sequence group of the planner's own
                    assert s == it["seq"] and shared[s] > 0
                assert it["key_end"] <= shared[s]
                rows += [(s, (tok - q_start[s]) * G + g) for g in range(G)]
        else:                          # decode/verify: up to 16 rows, or a row-split task of up to 48
            assert 1 <= it["row_count"] <= 48 and it["q_head"] == -1
            assert it["row_count"] <= 16 or it["row_begin"] % 48 == 0
            rows = [(it["seq"], r) for r in range(it["row_begin"], it["row_begin"] + it["row_count"])]
        for s, r in rows:
            seen.setdefault((s, it["kv_head"], r), []).append((it["key_begin"], it["key_end"], it["kind"],
                                                               it["split"], it["num_splits"]))
    for s, sp in enumerate(batch.seqs):
        for h in range(batch.num_kv_heads):
            for r in range(sp.query_len * G):
                rngs = sorted(seen.pop((s, h, r)))
                # contiguous, non-overlapping, starting at 0
                assert rngs[0][0] == 0
                for a, b in zip(rngs[:-1], rngs[1:]):
                    assert a[1] == b[0]
                # must reach this row's own position (the last key it may see)
                t = r // G
                assert rngs[-1][1] >= sp.seq_len - sp.query_len + t + 1
                assert rngs[-1][1] <= sp.seq_len
                casc = [x for x in rngs if x[2] == 2]
                own = [x for x in rngs if x[2] != 2]
                if casc and not own:   # tensor-core verify rows: cascade-kind chunks of all keys
                    assert s in _tc_verify_set(batch, head_dim, prefix_group, prefix_len)
                    assert all(x[4] == len(casc) for x in casc) and casc[-1][1] == sp.seq_len
                    assert sorted(x[3] for x in casc) == list(range(len(casc)))
                elif casc:             # cascade chunks then the sequence's own splits
                    assert all(x[4] == len(casc) for x in casc)
                    assert sorted(x[3] for x in casc) == list(range(len(casc)))
                    assert all(x[2] == 0 and x[4] == len(own) + len(casc) for x in own)
                    assert sorted(x[3] for x in own) == list(range(len(own)))
                    assert casc[-1][1] == own[0][0] == shared[s]
                else:
                    n = rngs[0][4]
                    assert len(rngs) == n and sorted(x[3] for x in rngs) == (list(range(n)) if n > 1 else [-1])
    assert not seen


@pytest.mark.parametrize("name", W.CONFIG_NAMES)
def test_planner_covers_configs(name):
    gen = __import__("torch").Generator().manual_seed(W.CONFIG_NAMES.index(name))
    seqs, Hq, Hkv, d, _ = W.config_seqs(name, gen)

    class B:  # structure only: no tensors needed for the planner
        pass
    b = B()
    b.seqs, b.num_q_heads, b.num_kv_heads = seqs, Hq, Hkv
    if name == "llama33_70b_prefill":
        b.seqs = seqs[:2]                       # keep the pure-Python coverage check fast
    pages = sum((s.seq_len + 15) // 16 for s in b.seqs)
    items = pk.inspect([s.seq_len for s in b.seqs], [s.query_len for s in b.seqs],
                       [s.mask_kind for s in b.seqs], [p for s in b.seqs for p in s.parents],
                       num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, num_pages=pages,
                       bt_stride=max((s.seq_len + 15) // 16 for s in b.seqs))
    _coverage(b, items, head_dim=d)
    # listed as launched: cascade tasks, prefill tasks, then decode/verify tasks (heaviest first)
    kinds = [it["kind"] for it in items]
    assert kinds == sorted(kinds, reverse=True)
    dec = [it for it in items if it["kind"] == 0]
    # heaviest first: pages, times 4 for a row-split task (more than 16 rows, every warp
    # runs every page)
    cost = [((it["key_end"] + 15) // 16 - it["key_begin"] // 16) * (4 if it["row_count"] > 16 else 1)
            for it in dec]
    assert cost == sorted(cost, reverse=True)
    assert all(it["key_end"] - it["key_begin"] <= 1024 * 16 for it in dec)


@pytest.mark.parametrize("seed, d, max_q", [(s, 64, 40) for s in range(4)] + [(s, 128, 300) for s in range(4, 8)])
def test_planner_covers_random_batches(seed, d, max_q):
    b = W.random_small(seed, num_seqs=6, d=d, max_ctx=300, max_q=max_q, tree_frac=0.4)
    items = pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat,
                       num_q_heads=b.num_q_heads, num_kv_heads=b.num_kv_heads, head_dim=b.head_dim,
                       num_pages=b.k_cache.shape[0], bt_stride=b.block_table.shape[1],
                       num_sms=4, ctas_per_sm=1)
    _coverage(b, items, head_dim=d)


def test_empty_batch_plans_to_nothing():
    assert pk.inspect([], [], [], num_q_heads=8, num_kv_heads=2, head_dim=64, num_pages=0,
                      bt_stride=0) == []


def test_long_context_is_split():
    items = pk.inspect([100000] * 2, [1, 1], [0, 0], num_q_heads=128, num_kv_heads=8,
                       head_dim=128, num_pages=12500, bt_stride=6250)
    assert all(it["num_splits"] > 1 for it in items)
    assert len(items) >= 148


def _shared_inspect(b, **kw):
    return pk.inspect(b.seq_lens, b.query_lens, b.mask_kinds, b.parents_flat, num_q_heads=b.num_q_heads,
                      num_kv_heads=b.num_kv_heads, head_dim=b.head_dim, num_pages=b.k_cache.shape[0],
                      bt_stride=b.block_table.shape[1], prefix_group=b.prefix_group,
                      prefix_len=b.prefix_len, **kw)


@pytest.mark.parametrize("seed, heads", [(0, (16, 4)), (1, (28, 4)), (2, (8, 8)), (3, (64, 2))])
def test_planner_covers_shared_prefix_batches(seed, heads):
    b = W.random_shared_small(seed, *heads)
    items = _shared_inspect(b, num_sms=4, ctas_per_sm=1)
    assert any(it["kind"] == 2 for it in items)
    _coverage(b, items, b.prefix_group, b.prefix_len, b.head_dim)


def test_planner_covers_shared_prefix_config():
    b = W.make_shared_config("llama3_8b_shared_prefix")
    items = _shared_inspect(b)
    _coverage(b, items, b.prefix_group, b.prefix_len, b.head_dim)
    casc = [it for it in items if it["kind"] == 2]
    # 4 groups x 8 KV heads x one task of 64 tokens x 2 chunks of 2048 shared keys
    assert len(casc) == 4 * 8 * 1 * 2


@pytest.mark.parametrize("groups, lens, code", [
    ([0, -1, 0], [16], -1),          # members not consecutive
    ([0, 0, -1], [24], -1),          # not a page multiple
    ([0, 0, -1], [48], -1),          # beyond the committed prefix of a member
    ([0, 2, -1], [16], -1),          # group id out of range
])
def test_planner_rejects_bad_groups(groups, lens, code):
    with pytest.raises(pk.PkvaError) as ei:
        pk.inspect([40, 60, 30], [1, 1, 1], [0, 0, 0], num_q_heads=8, num_kv_heads=2, head_dim=128,
                   num_pages=12, bt_stride=4, prefix_group=groups, prefix_len=lens)
    assert ei.value.code == code


def test_shared_prefix_and_prefill_tasks_at_head_dim_64():
    """Over bf16 caches the tensor-core tasks also run at head_dim 64: a shared-prefix group
    gets cascade tasks and a long causal chunk prefill tasks (FP8 plans keep them at 128,
    their staging copies being head_dim 128: the GPU tests check that refusal)."""
    items = pk.inspect([40, 60], [1, 1], [0, 0], num_q_heads=8, num_kv_heads=2, head_dim=64,
                       num_pages=12, bt_stride=4, prefix_group=[0, 0], prefix_len=[32])
    assert any(it["kind"] == 2 and it["key_end"] == 32 for it in items)
    items = pk.inspect([700, 40], [300, 1], [0, 0], num_q_heads=8, num_kv_heads=2, head_dim=64,
                       num_pages=50, bt_stride=44)
    assert any(it["kind"] == 1 for it in items)


@pytest.mark.parametrize("num_sms, ctas", [(1, 1), (4, 3), (148, 3)])
def test_decode_tasks_never_exceed_the_staged_block_table_slice(num_sms, ctas):
    """A decode/verify task stages its block-table entries in shared memory (1024 of them), so
    no task may span more pages, whatever the number of CTA slots the split targets."""
    lens = [200_000, 131_072, 16_385, 1024 * 16 + 1, 17]
    items = pk.inspect(lens, [1, 1, 1, 1, 1], [0] * 5, num_q_heads=16, num_kv_heads=2, head_dim=128,
                       num_pages=sum((L + 15) // 16 for L in lens), bt_stride=(max(lens) + 15) // 16,
                       num_sms=num_sms, ctas_per_sm=ctas)
    assert items and all(it["kind"] == 0 for it in items)
    for it in items:
        assert (it["key_end"] + 15) // 16 - it["key_begin"] // 16 <= 1024
    # every (sequence, KV head) still covers all its keys
    for s, L in enumerate(lens):
        for h in range(2):
            spans = sorted((it["key_begin"], it["key_end"]) for it in items if it["seq"] == s and it["kv_head"] == h)
            assert spans[0][0] == 0 and spans[-1][1] == L
            assert all(a[1] == b[0] for a, b in zip(spans[:-1], spans[1:]))



def _static_call(**over):
    """run_static on a 2-sequence batch whose tensors live on the host (CPU)."""
    import torch
    a = dict(seq_lens=[40, 17], query_lens=[8, 1], block_table=torch.zeros(2, 4, dtype=torch.int32),
             mask_kind=[W.CAUSAL, W.CAUSAL], parents=None,
             q=torch.zeros(9, 8, 64, dtype=torch.bfloat16), k_cache=torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16),
             v_cache=torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16), out=torch.zeros(9, 8, 64, dtype=torch.bfloat16),
             num_q_heads=8, num_kv_heads=2, head_dim=64, num_pages=8)
    a.update(over)
    return pk.run_static(a.pop("seq_lens"), a.pop("query_lens"), a.pop("block_table"), a.pop("mask_kind"),
                         a.pop("parents"), a.pop("q"), a.pop("k_cache"), a.pop("v_cache"), a.pop("out"), **a)


def _bt(dtype="int32", shape=(2, 4)):
    import torch
    return torch.zeros(*shape, dtype=getattr(torch, dtype))


@pytest.mark.parametrize("over, what", [
    (dict(query_lens=[8]), "one entry per sequence"),
    (dict(mask_kind=[W.CAUSAL]), "one entry per sequence"),
    (dict(seq_lens=[40, 17, 5]), "one entry per sequence"),
    (dict(block_table="host int32"), "block_table"),
    (dict(block_table="host int64"), "block_table"),
    (dict(block_table="numpy"), "block_table"),
])
def test_run_static_rejects_bad_host_arguments_before_the_call(over, what):
    # the binding checks what the C side cannot see (array lengths, where and what the
    # tensors are) and raises before it reaches the library, so no device is touched
    bt = over.get("block_table")
    if bt == "host int32":
        over["block_table"] = _bt("int32")
    elif bt == "host int64":
        over["block_table"] = _bt("int64")
    elif bt == "numpy":
        over["block_table"] = np.zeros((2, 4), dtype=np.int32)
    with pytest.raises(ValueError, match=what):
        _static_call(**over)


def test_verify_units_wider_than_32_rows_are_row_split_tasks_in_mixed_batches():
    """In a batch of mostly decode steps, a draft tree of 5 tokens under a GQA group of 7 has
    35 packed rows per KV head: one task reads its pages once (no 16-row chunks re-reading
    them); a 64-token tree under the same group (448 rows) becomes nine 48-row tasks and one
    16-row task; a tree of 20 rows stays two 16-row tasks. A batch made only of such trees
    keeps 16-row tasks throughout."""
    lens = [2000, 900, 700] + [3000] * 20
    qlens = [5, 64, 3] + [1] * 20
    kinds = [W.TREE, W.TREE, W.TREE] + [W.CAUSAL] * 20
    parents = [-1, 0, 0, 2, -1] + [-1] + list(range(63)) + [-1, 0, 1]
    pages = sum((L + 15) // 16 for L in lens)
    items = pk.inspect(lens, qlens, kinds, parents, num_q_heads=28, num_kv_heads=4, head_dim=64,
                       num_pages=pages, bt_stride=200)
    rows = sorted((it["seq"], it["kv_head"], it["row_begin"], it["row_count"]) for it in items
                  if it["kind"] == 0 and it["split"] <= 0)
    assert [r for r in rows if r[0] == 0] == [(0, h, 0, 35) for h in range(4)]
    big = [r[2:] for r in rows if r[0] == 1 and r[1] == 0]
    assert big == [(0, 48), (48, 48), (96, 48), (144, 48), (192, 48), (240, 48), (288, 48), (336, 48),
                   (384, 48), (432, 16)]
    assert [r[2:] for r in rows if r[0] == 2 and r[1] == 0] == [(0, 16), (16, 5)]
    only = pk.inspect(lens[:3], qlens[:3], kinds[:3], parents, num_q_heads=28, num_kv_heads=4, head_dim=64,
                      num_pages=pages, bt_stride=200)
    assert max(it["row_count"] for it in only if it["kind"] == 0) == 16


def test_verify_trees_run_as_tensor_core_tasks():
    """Beside decode steps, a tree of 17 to 128 packed rows per KV head with at least 512 keys
    runs as cascade-kind tensor-core tasks over all of its keys, one per KV head and chunk of
    32 KV tiles (4096 keys), with no decode/verify task. A 64-token tree (448 rows), a tree of
    16 rows or fewer, fewer than 512 keys, head_dim 64, and members of the caller's
    shared-prefix groups keep the decode/verify path (a group member's shared prefix stays a
    cascade task); so does every tree of a batch where such trees hold more than half of the
    decode/verify pages."""
    lens = [2000, 900, 700, 3000, 400, 5000] + [3000] * 10
    qlens = [5, 64, 3, 2, 5, 5] + [1] * 10
    kinds = [W.TREE] * 6 + [W.CAUSAL] * 10
    parents = [-1, 0, 0, 2, -1] + [-1] + list(range(63)) + [-1, 0, 1] + [-1, 0] + [-1, 0, 0, 2, -1] + [-1, 0, 1, 1, 0]
    pages = sum((L + 15) // 16 for L in lens)
    kw = dict(num_q_heads=28, num_kv_heads=4, num_pages=pages, bt_stride=400)
    items = pk.inspect(lens, qlens, kinds, parents, head_dim=128, **kw)
    casc = sorted((it["seq"], it["kv_head"], it["key_begin"], it["key_end"], it["row_count"], it["split"],
                   it["num_splits"]) for it in items if it["kind"] == 2)
    split5 = [(0, 2560, 0), (2560, 5000, 1)]                      # 40 tiles in two chunks
    assert casc == [(0, h, 0, 2000, 5, 0, 1) for h in range(4)] + [(2, h, 0, 700, 3, 0, 1) for h in range(4)] + \
        [(5, h, kb, ke, 5, k, 2) for h in range(4) for kb, ke, k in split5]
    assert not any(it["kind"] == 0 and it["seq"] in (0, 2, 5) for it in items)
    assert {it["seq"] for it in items if it["kind"] == 0} == {1, 3, 4} | set(range(6, 16))
    assert not any(it["kind"] == 2 for it in pk.inspect(lens, qlens, kinds, parents, head_dim=64, **kw))
    grouped = pk.inspect(lens, qlens, kinds, parents, head_dim=128, prefix_group=[0] + [-1] * 15, prefix_len=[512],
                         **kw)
    assert sorted({(it["seq"], it["key_end"]) for it in grouped if it["kind"] == 2}) == \
        [(0, 512), (2, 700), (5, 2560), (5, 5000)]
    assert min(it["key_begin"] for it in grouped if it["kind"] == 0 and it["seq"] == 0) == 512
    # the trees alone: more than half of the pages, so all stay on the decode/verify path
    alone = pk.inspect(lens[:6], qlens[:6], kinds[:6], parents, head_dim=128, **kw)
    assert not any(it["kind"] == 2 for it in alone)
