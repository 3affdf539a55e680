"""GPU parity of shared-prefix (cascade) plans (attn_plan_shared): sequences that share
their first keys get those keys' contribution from cascade tasks (stacked (token, head)
rows on tensor-core tiles) and merge it with their own keys' partial results.

Checked: every row against the float64 oracle (which reads each sequence's full K/V), the
same batch planned without groups, repeated runs (the arrival counters reset), and the
fused append on a shared plan.
"""
import pytest
import torch

import paged_kv_attention_verify_b200 as pk
import workloads as W
from _util import assert_close, oracle_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("seed, heads", [(0, (16, 4)), (1, (28, 4)), (2, (8, 8)), (3, (64, 2)), (4, (32, 1))])
def test_shared_prefix_small_all_rows(seed, heads, d):
    b = W.random_shared_small(seed, *heads, device=DEV, d=d)
    plan = pk.plan_for_batch(b)
    assert plan.info()["num_cascade_items"] > 0
    out = plan.run(b.q, b.k_cache, b.v_cache)
    assert plan.check() == 0
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, f"shared prefix seed {seed}")
    again = plan.run(b.q, b.k_cache, b.v_cache)
    assert plan.check() == 0
    assert torch.equal(bits(out), bits(again)), "a second run of the plan differs"
    plain = pk.plan_for_batch(b, shared=False)
    ref = plain.run(b.q, b.k_cache, b.v_cache)
    assert plain.check() == 0
    assert (out.float() - ref.float()).abs().max().item() <= 2e-2
    plan.close()
    plain.close()


def _sample(sp):
    return sorted({0, sp.query_len - 1})


def test_shared_prefix_config_full_size():
    b = W.make_shared_config("llama3_8b_shared_prefix", device=DEV)
    plan = pk.plan_for_batch(b)
    info = plan.info()
    assert info["num_cascade_items"] == 4 * 8 * 2
    out = plan.run(b.q, b.k_cache, b.v_cache)
    assert plan.check() == 0
    seq_ids = list(range(0, len(b.seqs), 5))
    rows, exp = oracle_rows(b, seq_ids=seq_ids, token_picker=_sample)
    assert_close(out[rows], exp, "llama3_8b_shared_prefix")
    plain = pk.plan_for_batch(b, shared=False)
    assert plain.info()["kv_bytes"] > 5 * info["kv_bytes"]      # 4096 shared keys vs ~512 own
    ref = plain.run(b.q, b.k_cache, b.v_cache)
    assert plain.check() == 0
    assert (out.float() - ref.float()).abs().max().item() <= 2e-2
    plan.close()
    plain.close()


@pytest.mark.parametrize("d", [128, 64])
def test_shared_prefix_with_fused_append(d):
    b = W.random_shared_small(5, 16, 4, device=DEV, d=d)
    k_new, v_new = W.new_token_kv(b)
    pg, sl = W.new_token_slots(b)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    kc[pg, :, sl] = float("nan")
    vc[pg, :, sl] = float("nan")
    plan = pk.plan_for_batch(b)
    out = plan.run_append(b.q, k_new, v_new, kc, vc)
    assert plan.check() == 0
    assert torch.equal(bits(kc), bits(b.k_cache)) and torch.equal(bits(vc), bits(b.v_cache))
    rows, exp = oracle_rows(b)
    assert_close(out[rows], exp, "shared prefix + append")
    plan.close()
