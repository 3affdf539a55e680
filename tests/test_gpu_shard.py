"""GPU: a batch split over `world` GPUs (KV-head groups x sequence subsets, no exchange in
attention) gives the whole batch's result. The ranks run one after another on the one GPU
here; each shard is planned and run through the C ABI exactly as its own GPU would."""
import numpy as np
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, oracle_rows
from paged_kv_attention_verify_b200 import shard as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_sharded(b, world):
    out = torch.zeros_like(b.q)
    qo = b.q_offsets()
    for r in range(world):
        part = W.shard_batch(b, r, world)
        if not part.seqs:
            continue
        tpr, spr, tp, sp = S.shard_coords(r, world, b.num_kv_heads)
        kv0, kv1, q0, q1 = S.head_range(tpr, tp, b.num_q_heads, b.num_kv_heads)
        plan = pk.plan_for_batch(part)
        res = plan.run(part.q, part.k_cache, part.v_cache)
        assert plan.check() == 0
        row = 0
        for s in S.sequence_subset(len(b.seqs), spr, sp):
            T = b.seqs[s].query_len
            out[qo[s]:qo[s] + T, q0:q1] = res[row:row + T]
            row += T
        plan.close()
    return out


@pytest.mark.parametrize("world", [2, 4, 8])
def test_sharded_small_batch(world):
    b = W.random_small(43, num_seqs=6, Hq=16, Hkv=4, d=128, max_ctx=400, max_q=80, tree_frac=0.3, device=DEV)
    out = run_sharded(b, world)
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, f"sharded over {world}")


@pytest.mark.parametrize("world", [2, 8])
def test_sharded_unified_config(world):
    b = W.make_config("qwen2_7b_unified", device=DEV)
    out = run_sharded(b, world)
    whole = pk.plan_for_batch(b)
    ref = whole.run(b.q, b.k_cache, b.v_cache)
    assert whole.check() == 0
    assert (out.float() - ref.float()).abs().max().item() <= 2e-2
    rows, exp = oracle_rows(b, seq_ids=list(range(0, len(b.seqs), 11)), token_picker=lambda sp: [0, sp.query_len - 1])
    assert_close(out[rows], exp, f"unified sharded over {world}")
    whole.close()
